/*
 * mono.h -- C-ABI of the B200 (sm_100a) Monodratic mixer library.
 *
 * The library computes the forward pass of the stateless
 * [batch, sequence, width] -> attention-delta mixer described on the
 * aitechinspire.com Monodratic article ("Snapshot: key facts from the
 * report"): Q/K/V projection with RoPE, learned product-hash routing of
 * source blocks through bounded causal posting lists, exact causal softmax
 * over the selected token set, and the output projection.  Normalisation,
 * residuals and feed-forward layers stay with the host model.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensors are contiguous and row-major.  Device pointers point to
 *   global memory of the current CUDA device; `stream` is a cudaStream_t
 *   (NULL = the legacy default stream).
 * - Storage type: x, weights, Q, K, V, O and delta use cfg.dtype
 *   (MONO_F32 = IEEE binary32, MONO_BF16 = bfloat16).  Codebooks and the
 *   block summaries are always fp32; ids are int32.
 * - Layouts:
 *     x, delta        [B, S, W]
 *     Wq, Wk, Wv      [H*d, W]   out_features x in_features: q = x Wq^T,
 *                                head h owns rows h*d .. h*d+d-1
 *     Wo              [W, H*d]   delta = O Wo^T
 *     codebooks       [H, M, C, d/M] fp32
 *     Q, K, V         [B, H, S, d]   (Q and K after RoPE)
 *     sel             [B, H, S, R] int32, ascending block ids, -1 padding
 *     O               [B, S, H*d]    head h in columns h*d .. h*d+d-1
 *     forced          [B, H, S] int32 block id per query-head, -1 = none
 * - Ownership: the caller allocates every device buffer, including the
 *   workspace whose size mono_plan reports.  The library never allocates
 *   device memory and keeps no state between calls; a plan is immutable
 *   host data.
 * - Every device pointer must be 16-byte aligned and the workspace
 *   256-byte aligned (MONO_ERR_ALIGN otherwise).
 * - Calls are asynchronous on `stream`.  Argument errors are reported by
 *   the return code before anything is launched.  Errors that only the
 *   device can see are recorded in a device error word in the workspace and
 *   reported by mono_stats (MONO_ERR_DEVICE).  Nothing crosses the C
 *   boundary by exception.
 * - A call with B == 0 or S == 0 is valid and launches nothing.
 */
#ifndef MONO_H
#define MONO_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MONO_VERSION 1

enum mono_dtype { MONO_F32 = 0, MONO_BF16 = 1 };

enum mono_status {
    MONO_OK = 0,
    MONO_ERR_INVALID = 1,     /* parameters violate the method's definition (e.g. S % Bs != 0, R > E, T > C^M) */
    MONO_ERR_UNSUPPORTED = 2, /* valid, but outside what this build implements (e.g. d not in {64, 128}) */
    MONO_ERR_NULL = 3,        /* a required pointer is NULL */
    MONO_ERR_WORKSPACE = 4,   /* workspace pointer missing */
    MONO_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
    MONO_ERR_DEVICE = 6,      /* a kernel recorded an error in the device error word */
    MONO_ERR_ALIGN = 7,       /* a pointer is not suitably aligned */
    MONO_ERR_SCRATCH = 8      /* the problem needs more than mono_route_static's fixed scratch array */
};

/* Plan options (mono_config.flags). */
enum mono_flags {
    /* Run the plain kernels (SIMT projections, query-major SIMT attention)
     * even where the tensor-core kernels apply.  Same results within the
     * stated tolerances; used as the correctness baseline.  The tensor-core
     * kernels apply to bf16 storage with: projections W % 128 == 0 and
     * H*d % 128 == 0; attention Bs in {64, 128} and 128 + (L-1)*Bs <= 256. */
    MONO_FLAG_SIMPLE_KERNELS = 1,
    /* Redirect-on-overflow instead of drop (remio.ai article, the section on
     * retrieval decisions: a strict capacity bounds each list, and overflow
     * handling may drop or redirect blocks; the pages give no rule).  A block
     * whose own list is full goes to the first list with room among the next
     * addresses in mixed-radix order (a+1, a+2, ... mod C^M); it is dropped,
     * and counted in the overflow, only when every list is full.  The posting
     * export lists blocks under the address of the list that holds them, the
     * dropped ones last under the address C^M.  Needs C^M <= 65536; not
     * available to the decode entry points (MONO_ERR_UNSUPPORTED). */
    MONO_FLAG_REDIRECT = 2
};

/* Shape and method parameters.  Symbols follow the pages' description:
 * B batch, S sequence, W width, H heads, d head dim, Bs block size,
 * L guaranteed local blocks, R remote blocks kept, E eligible candidates
 * reranked, M subspaces, C codes per subspace (C^M product addresses),
 * T probed addresses, cap posting-list capacity. */
typedef struct mono_config {
    int B, S, W, H, d;
    int Bs, L, R, E, M, C, T, cap;
    double rope_theta;
    int dtype; /* enum mono_dtype */
    int flags; /* enum mono_flags */
} mono_config;

typedef struct mono_plan_s mono_plan_t;

/* Routing statistics of the last mono_route / mono_forward on a workspace
 * (the quantities the pages ask to log: selected remote blocks per query
 * and posting overflow counts). */
typedef struct mono_stats {
    int64_t overflow_total;    /* blocks dropped from full posting lists, all (b, h) */
    int32_t overflow_max_bh;   /* largest per-(b, h) overflow */
    int32_t device_error;      /* 0, or the first device error code recorded: 1 a sel id outside
                                  [0, t/Bs - L], 2 probe candidate bound exceeded, 3 a bounded
                                  wait ran out, 4 an address outside [0, C^M), 5 shared memory
                                  not 1024-byte aligned */
    int64_t queries_lt_R;      /* query-heads that received fewer than R remote blocks */
    int64_t remote_selected;   /* total remote blocks selected */
    double mean_remote;        /* remote_selected / (B*H*S) */
    int64_t forced_ignored;    /* forced ids that were not eligible */
    int64_t probe_walks;       /* query-heads whose exact top-T left the probe's fast path for the general
                                  walk (near ties); the first 4096 are listed in MONO_WS_WALK_LOG */
} mono_stats_t;

/* Workspace regions that mono_workspace_region can locate (debug/export). */
enum mono_ws_region {
    MONO_WS_KBAR = 0,      /* [B,H,nb,d] fp32 block summaries */
    MONO_WS_ADDR = 1,      /* [B,H,nb] int32 product address of each block */
    MONO_WS_POST_IDS = 2,  /* [B,H,nb] int32 block ids sorted by (address, id) */
    MONO_WS_POST_ADDR = 3, /* [B,H,nb] int32 address of each sorted entry */
    MONO_WS_POST_RANK = 4, /* [B,H,nb] int32 position within its address; kept iff < cap */
    MONO_WS_OVERFLOW = 5,  /* [B,H] int32 dropped blocks */
    MONO_WS_Q = 6,         /* [B,H,S,d] dtype, used by mono_forward */
    MONO_WS_K = 7,
    MONO_WS_V = 8,
    MONO_WS_SEL = 9,       /* [B,H,S,R] int32, used by mono_forward */
    MONO_WS_O = 10,        /* [B,S,H*d] dtype, used by mono_forward */
    MONO_WS_WALK_LOG = 11, /* [4096] int32: flat indices (b*H+h)*S+t of the first query-heads whose probe took the
                              general walk (mono_stats.probe_walks of them; unspecified order) */
    MONO_WS_NREGIONS = 12
};

/* Validate `cfg` and build an immutable host-side plan.  Writes the
 * workspace size in bytes the plan's calls need.  No device work.
 * The parameters are those of the mixer the aitechinspire.com article
 * describes ("Snapshot: key facts from the report": blocks, bounded causal
 * posting lists, probed product addresses, a fixed number R of remote
 * blocks plus guaranteed local blocks); the validity rules are the method's
 * definition (S a whole number of blocks, R <= E, T <= C^M, cap >= 1, ...).
 * `cfg` is read, not kept.  `*plan` is owned by the caller (free it with
 * mono_plan_destroy); it is NULL on any error.
 * Returns MONO_OK, MONO_ERR_NULL, MONO_ERR_INVALID or MONO_ERR_UNSUPPORTED. */
int mono_plan(const mono_config *cfg, mono_plan_t **plan, size_t *workspace_bytes);

/* Free a plan (NULL is ignored). */
void mono_plan_destroy(mono_plan_t *plan);

/* Byte offset and size of a workspace region (see enum mono_ws_region). */
int mono_workspace_region(const mono_plan_t *plan, int region, size_t *offset, size_t *bytes);

/* Q/K/V projection + RoPE (aitechinspire.com article, Snapshot: after RoPE,
 * source blocks are assigned to posting lists).  q = x Wq^T etc., no bias;
 * RoPE rotates interleaved pairs (2i, 2i+1) of Q and K by t*theta^(-2i/d).
 * Inputs x, Wq, Wk, Wv; outputs Q, K, V.  Uses the workspace for the
 * rotation tables. */
int mono_project(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk,
                 const void *Wv, void *Q, void *K, void *V, void *workspace, void *stream);

/* Learned product-hash routing ("Monodratic Routes Sparse Attention with
 * Learned Product Hashes", Key Points; remio.ai article section on
 * retrieval decisions): block summaries kbar (mean post-RoPE key), product
 * address by per-subspace dot-product argmax, bounded causal posting lists
 * (earliest cap blocks kept, the rest dropped and counted), per-query probe
 * of the top-T product addresses, union of their lists filtered to blocks
 * j <= t/Bs - L and capped at E, rerank by q.kbar keeping the top R.
 * Integer decisions use fp32 with the fixed accumulation order of the
 * specification, so results are deterministic.
 * Inputs Q, K, codebooks; optional `forced` (NULL = none): an eligible
 * forced block replaces the lowest-ranked selection (or is appended) so the
 * count stays <= R.  Output sel.  Summaries, addresses, posting lists and
 * overflow counts are left in the workspace (mono_workspace_region). */
int mono_route(const mono_plan_t *plan, const void *Q, const void *K, const float *codebooks,
               const int32_t *forced, int32_t *sel, void *workspace, void *stream);

/* The three stages of mono_route, callable one at a time (same kernels,
 * same results); each reads what the previous one left in the workspace.
 *  - mono_route_summaries: block summaries kbar and product addresses (needs K).
 *  - mono_route_lists:     bounded causal posting lists and overflow counts;
 *                          resets the routing statistics.
 *  - mono_route_queries:   probe, union, causal filter, E cap, rerank -> sel
 *                          (needs Q); also resets and fills the statistics.
 * The lists kernel is launched so that it may start while the summaries
 * kernel before it on the stream still runs, and the probe so that it may
 * start while the lists kernel runs (programmatic dependent launch): each
 * waits for its predecessor before reading what that one writes, so the
 * probe loads its queries and scores the codebooks meanwhile.
 * mono_route_summaries resets the device error word. */
int mono_route_summaries(const mono_plan_t *plan, const void *K, const float *codebooks, void *workspace,
                         void *stream);
int mono_route_lists(const mono_plan_t *plan, void *workspace, void *stream);
int mono_route_queries(const mono_plan_t *plan, const void *Q, const float *codebooks, const int32_t *forced,
                       int32_t *sel, void *workspace, void *stream);

/* mono_route without a workspace, for callers that cannot allocate device
 * memory (a plugin whose host framework owns every device allocation, or a
 * serving loop that forbids cudaMalloc after start-up).  There is no
 * counterpart on the pages: this is a deployment convenience of this library.
 * Same kernels and same results as mono_route; inputs Q, K, codebooks,
 * optional forced; output sel.  The routing tables live in one array of
 * mono_route_static_capacity() bytes (16 MiB) that the library places in the
 * global memory of every GPU it is loaded on, for the life of the process.
 * The tables need B*H*nb*(4*d + 16) + B*H*4 + 64 bytes, each of the seven
 * regions rounded up to 256 bytes (kbar is fp32); a larger problem returns
 * MONO_ERR_SCRATCH before anything is launched.
 * The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current) and caches it, so make
 * the first call on each device before any stream capture.  All calls on a
 * device share the array: calls that overlap on the GPU (other streams or
 * threads) race and must be serialised by the caller.  Each call clears the
 * statistics counters it uses and overwrites the tables; mono_stats with a
 * NULL workspace reads them back.  The cached address is not valid across
 * cudaDeviceReset: do not call this entry point on a device after resetting
 * it in the same process.  No memory is allocated by this entry point. */
int mono_route_static(const mono_plan_t *plan, const void *Q, const void *K, const float *codebooks,
                      const int32_t *forced, int32_t *sel, void *stream);

/* Size in bytes of the fixed array behind mono_route_static. */
size_t mono_route_static_capacity(void);

/* Exact causal softmax over the selected token set (aitechinspire.com
 * article, Snapshot): for query t of block bq, the tokens of the blocks in
 * sel[t] plus the tokens s in [max(0, bq-L+1)*Bs, t], scale 1/sqrt(d),
 * softmax in fp32 with fp32 accumulation.  Inputs Q, K, V, sel; output O.
 * sel entries must be -1 or a block id <= t/Bs - L (out-of-range ids are
 * skipped and recorded in the device error word). */
int mono_attend(const mono_plan_t *plan, const void *Q, const void *K, const void *V,
                const int32_t *sel, void *O, void *workspace, void *stream);

/* The stages of mono_attend, callable one at a time (same kernels, same
 * results): with the tensor-core kernels (bf16, see MONO_FLAG_SIMPLE_KERNELS)
 *  - mono_attend_pairs:  the (query, remote block) pairs of sel grouped by
 *                        block into work items, in the workspace;
 *  - mono_attend_remote: one partial softmax (normalised output in bf16, its
 *                        max and sum) per pair, block by block, in the
 *                        workspace;
 *  - mono_attend_local:  the local part of every query tile and the exact
 *                        merge with its remote partials -> O.
 * With the plain kernels the whole attention is one query-major kernel,
 * which mono_attend_local runs; the other two do nothing.  Each stage reads
 * what the previous one left in the workspace. */
int mono_attend_pairs(const mono_plan_t *plan, const int32_t *sel, void *workspace, void *stream);
int mono_attend_remote(const mono_plan_t *plan, const void *Q, const void *K, const void *V, void *workspace,
                       void *stream);
int mono_attend_local(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel,
                      void *O, void *workspace, void *stream);

/* Output projection delta = O Wo^T: the last step of the stateless
 * [batch, sequence, width] -> attention-delta mixer (aitechinspire.com
 * article, "Snapshot: key facts from the report"; the host model adds the
 * residual).  O [B,S,H*d] and Wo [W,H*d] in dtype; delta [B,S,W] in dtype,
 * rounded once from the fp32 accumulation.  The workspace holds the device
 * error word that a bounded wait of the tensor-core kernel may set. */
int mono_out_project(const mono_plan_t *plan, const void *O, const void *Wo, void *delta,
                     void *workspace, void *stream);

/* ------------------------------------------------------------------------
 * Head-sharded mixer on several GPUs (one process per GPU): rank r of N runs
 * a plan of H/N heads (its rows of Wq, Wk, Wv, its columns of Wo, its
 * codebooks).  The mixer's output delta = sum over heads of O_h Wo_h^T (the
 * output projection of the aitechinspire.com article's attention-delta
 * mixer, "Snapshot: key facts from the report") is then a sum of the ranks'
 * partials, taken as a reduce-scatter over token rows: the B*S rows are
 * split into N equal chunks, chunk c owned by rank c.
 *  - mono_out_project_scatter: the rank's output projection, its fp32 rows
 *    written by the GEMM epilogue straight into the owners' staging buffers
 *    (stage[c]: rank c's buffer, [N][B*S/N][W] fp32, this rank's partial at
 *    slot `rank`; pointers of other GPUs' memory reachable by peer access,
 *    e.g. symmetric memory over NVLink).  No partial is rounded to bf16.
 *  - mono_stage_reduce: after every rank's scatter has completed (the caller
 *    orders this, e.g. with a collective on the stream), the owner sums its N
 *    staged partials in fp32 in ascending rank order and rounds once:
 *    delta_chunk [B*S/N][W] bf16 = rows c*B*S/N .. of delta.
 * bf16 storage with the tensor-core projections only (MONO_ERR_UNSUPPORTED
 * otherwise); 1 <= N <= 8 with (B*S) % N == 0 (MONO_ERR_INVALID).
 * ------------------------------------------------------------------------ */
int mono_out_project_scatter(const mono_plan_t *plan, const void *O, const void *Wo, float *const *stage,
                             int nranks, int rank, void *workspace, void *stream);
int mono_stage_reduce(const mono_plan_t *plan, const float *stage, int nranks, void *delta_chunk, void *stream);

/* The whole mixer (aitechinspire.com article, "Snapshot: key facts from
 * the report" and "What's the core idea?": after RoPE, blocks go to bounded
 * causal posting lists; each query probes product addresses, reranks,
 * selects R remote blocks, adds its guaranteed local blocks and runs exact
 * causal softmax over those tokens; the stateless mixer returns an attention
 * delta): mono_project, mono_route, mono_attend and mono_out_project on
 * workspace-resident Q, K, V, sel and O.  Inputs x [B,S,W], weights,
 * codebooks, optional forced; output delta [B,S,W].  The workspace keeps
 * every intermediate (mono_workspace_region) for mono_stats and debugging. */
int mono_forward(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk,
                 const void *Wv, const void *Wo, const float *codebooks, const int32_t *forced,
                 void *delta, void *workspace, void *stream);

/* ------------------------------------------------------------------------
 * Decode: one new token per sequence against caller-owned caches.
 *
 * The pages describe the batch forward only.  Every stage of it is causal
 * (the posting lists keep the earliest `cap` blocks of each address, so a
 * list at position t holds exactly the blocks a streaming build would hold),
 * hence step t of the decode computes row t of mono_forward on the first t+1
 * tokens: same projection, same routing decisions on the same Q/K values,
 * same selected token set.  The incremental parts are the append of a block
 * that position t completes to its posting list, and a single-query
 * route + attend over the cache.
 *
 * The cache is one caller-allocated device buffer of mono_decode_cache_bytes
 * bytes, for the plan's B, H and S (S = the largest context).  Its regions
 * (enum mono_dec_region, located by mono_decode_cache_region):
 * ------------------------------------------------------------------------ */
enum mono_dec_region {
    MONO_DEC_K = 0,        /* [B,H,S,d] dtype post-RoPE keys (the layout of mono_project's K) */
    MONO_DEC_V = 1,        /* [B,H,S,d] dtype values */
    MONO_DEC_KBAR = 2,     /* [B,H,nb,d] fp32 summaries of completed blocks */
    MONO_DEC_ADDR = 3,     /* [B,H,nb] int32 product address of completed blocks */
    MONO_DEC_COUNT = 4,    /* [B,H,A] int32 blocks that reached each address (kept: the first cap) */
    MONO_DEC_HEAD = 5,     /* [B,H,A] int32 first kept block of each address, -1 if none */
    MONO_DEC_TAIL = 6,     /* [B,H,A] int32 last kept block of each address */
    MONO_DEC_NEXT = 7,     /* [B,H,nb] int32 next kept block of the same address, -1 at the end */
    MONO_DEC_OVERFLOW = 8, /* [B,H] int32 blocks dropped from full lists */
    MONO_DEC_Q = 9,        /* [B,H,d] dtype this step's post-RoPE query */
    MONO_DEC_SEL = 10,     /* [B,H,R] int32 this step's remote blocks, ascending, -1 padded */
    MONO_DEC_O = 11,       /* [B,H*d] dtype this step's attention output */
    MONO_DEC_NREGIONS = 12
};

/* Size of the decode cache.  MONO_ERR_UNSUPPORTED if C^M > 4096. */
int mono_decode_cache_bytes(const mono_plan_t *plan, size_t *bytes);

/* Byte offset and size of a decode-cache region. */
int mono_decode_cache_region(const mono_plan_t *plan, int region, size_t *offset, size_t *bytes);

/* Start from a context of t0 tokens (0 <= t0 <= S) whose keys and values the
 * caller has already written to the cache's K and V regions for positions
 * < t0 (e.g. copied from mono_project's K and V): computes the summaries and
 * addresses of the t0/Bs completed blocks (same arithmetic as
 * mono_route_summaries) and builds their posting lists in ascending block
 * order.  t0 = 0 empties the lists. */
int mono_decode_prefill(const mono_plan_t *plan, int t0, const float *codebooks, void *cache, void *stream);

/* One decode step at position t (steps in order t0, t0+1, ...; t < S).
 * x_t [B,W] and delta_t [B,W] (dtype); weights as for mono_project and
 * mono_out_project; forced_t [B,H] int32 or NULL (-1 = none), with the
 * meaning it has in mono_route.  The stages, callable one at a time:
 *  - mono_decode_project: q, k, v of x_t with RoPE at position t; q to the
 *    cache's Q region, k and v appended to K and V at position t;
 *  - mono_decode_route:   if t completes block j = t/Bs (t % Bs == Bs-1), its
 *    summary and address and the append to its posting list (or the
 *    overflow count); then the routing of the cache's Q: probe of the top-T
 *    product addresses, union in probe order, blocks j <= t/Bs - L, E cap,
 *    rerank by q.kbar, forced block -> the cache's SEL region;
 *  - mono_decode_attend:  exact softmax of the cache's Q over the tokens of
 *    the SEL blocks and the local tokens [max(0, t/Bs-L+1)*Bs, t] -> the
 *    cache's O region (fp32 scores and accumulation);
 *  - mono_decode_step:    the three, then delta_t = O Wo^T.
 * Routing decisions use the fp32 order of mono_route, so for equal Q and K
 * values the selections equal mono_route's row t. */
int mono_decode_project(const mono_plan_t *plan, int t, const void *x_t, const void *Wq, const void *Wk,
                        const void *Wv, void *cache, void *stream);
int mono_decode_route(const mono_plan_t *plan, int t, const float *codebooks, const int32_t *forced_t, void *cache,
                      void *stream);
int mono_decode_attend(const mono_plan_t *plan, int t, void *cache, void *stream);
int mono_decode_step(const mono_plan_t *plan, int t, const void *x_t, const void *Wq, const void *Wk,
                     const void *Wv, const void *Wo, const float *codebooks, const int32_t *forced_t,
                     void *delta_t, void *cache, void *stream);

/* ------------------------------------------------------------------------
 * Backward pass for a fixed selection.
 *
 * The routing (summaries, addresses, posting lists, probe, rerank) is
 * piecewise constant in its inputs and has no gradient; the selection sel
 * (e.g. from mono_route) is an input and the rest of the forward pass is
 * differentiated: projection, RoPE, exact softmax over the selected token set
 * of each query (the blocks of sel that lie in [0, t/Bs - L] plus the local
 * tokens [max(0, t/Bs - L + 1) * Bs, t]), output projection.  Gradients are
 * fp32 and accumulated in fp32, every sum in a fixed order (the queries that
 * selected a block in ascending order, a query's remote blocks in slot order,
 * split-K partial products in range order), so two calls on the same inputs
 * give the same bits.  With bf16 storage, Bs = 64 and d = 64 with L <= 2 or
 * d = 128 with L = 1, mono_backward runs the attention gradients on the tensor
 * cores with every operand given to 16 significant bits (bf16 hi + lo terms).
 * The backward workspace is a separate
 * caller-allocated buffer of mono_backward_workspace_bytes bytes (256-byte
 * aligned).
 * ------------------------------------------------------------------------ */
int mono_backward_workspace_bytes(const mono_plan_t *plan, size_t *bytes);

/* Gradients of the selected-set attention O(Q, K, V; sel) given dO:
 * Q, K, V [B,H,S,d] (dtype, post-RoPE, as mono_attend takes them), sel
 * [B,H,S,R], dO [B,S,H*d] fp32 -> dQ, dK, dV [B,H,S,d] fp32 (with respect to
 * the post-RoPE Q and K). */
int mono_attend_backward(const mono_plan_t *plan, const void *Q, const void *K, const void *V, const int32_t *sel,
                         const float *dO, float *dQ, float *dK, float *dV, void *bwd_workspace, void *stream);

/* Gradients of the whole mixer for a fixed selection: inputs as mono_forward
 * (x, Wq, Wk, Wv, Wo in dtype) plus sel [B,H,S,R] and ddelta [B,S,W] (dtype);
 * outputs dx [B,S,W] and dWq, dWk, dWv [H*d,W], dWo [W,H*d], fp32.  The forward
 * activations Q, K, V and O are recomputed into `workspace` (the forward
 * workspace of the plan).  With bf16 storage the five projection gradients
 * run on the tensor cores with bf16 operands: the stored activations and
 * weights and ddelta, which are bf16 already, and the fp32 gradients before
 * the projections (dQ, dK after the inverse rotation, dV), each given as two
 * bf16 terms hi + lo (16 significant bits); products accumulate in fp32.
 * With fp32 storage every operand stays fp32. */
int mono_backward(const mono_plan_t *plan, const void *x, const void *Wq, const void *Wk, const void *Wv,
                  const void *Wo, const int32_t *sel, const void *ddelta, float *dx, float *dWq, float *dWk,
                  float *dWv, float *dWo, void *workspace, void *bwd_workspace, void *stream);

/* Synchronise `stream` and read the routing statistics and the device error
 * word of the last mono_route / mono_forward on `workspace`: the quantities
 * the aitechinspire.com article ("Practical notes for tinkerers") asks a user
 * to log next to accuracy -- selected remote blocks per query and posting
 * overflow counts.  With workspace == NULL the statistics and error word of
 * the last mono_route_static call on the current device are read instead
 * (from that entry point's fixed array, with the same plan).  `out` is
 * caller-owned host memory.  Returns MONO_ERR_DEVICE if a kernel recorded an
 * error. */
int mono_stats(const mono_plan_t *plan, const void *workspace, void *stream, mono_stats_t *out);

/* Static description of a status code. */
const char *mono_strerror(int status);

/* MONO_VERSION of the built library. */
int mono_version(void);

/* Number of CUDA kernels this library has launched in this process (all
 * devices and streams).  Host-side counter; no device work. */
unsigned long long mono_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* MONO_H */
