/*
 * ep.h -- C ABI of the B200 expert-parallel dispatch library (libep.so).
 *
 * The hot path of an expert-parallel MoE layer whose ranks are balanced by
 * online redundant experts, with the R expert-parallel ranks simulated as R
 * partitions of one static buffer on one GPU:
 *
 *   ep_route_stats -> ep_plan -> ep_layout -> ep_dispatch -> (expert) -> ep_combine
 *   ep_align_sort (block-aligned expert sort for a grouped GEMM)
 *   ep_replica_grad_reduce (backward: replica gradients into the home expert)
 *   ep_route_fused (stats, plan, layout and align-sort in one launch)
 *   ep_route_dispatch_fused (the same, with dispatch, in one launch)
 *   ep_dispatch_backward, ep_combine_backward (gradients of the row movers)
 *   ep_prefetch_slots (a per-rank replica slot budget B applied to a plan)
 *   ep_quota_route, ep_quota_replica_grad_reduce (the quota-driven planner:
 *       a searched load threshold with at most B replicas per rank)
 *   rank-local form, one rank per process (ep_plan_from_counts,
 *       ep_layout_rank, ep_dispatch_peer, ep_combine_peer,
 *       ep_replica_grad_reduce_peer and their quota-planner counterparts;
 *       ep_ipc_export / ep_ipc_open / ep_ipc_close map peer buffers across
 *       processes)
 *   ep_route_stats_noalloc (ep_route_stats with the library's own scratch)
 *
 * Sources, cited by page title and section:
 *  [GR] "MoonEP: πώς η εξισορρόπηση των AI experts αλλάζει την υποδομή των MoE
 *       μοντέλων" (twodots.gr)
 *  [FR] "Moonshot AI открыла код MoonEP — библиотеки для обучения MoE-модели
 *       Kimi K3" (news.hamidun.com)
 *  [ZH] the MoE Align & Sort report (新智元报道, los70adestajo.com page)
 *  [JA] "Xiaohongshuと北京大学がUltraEPを発表、静的MoE負荷分散に挑戦" (remio.ai)
 *
 * Notation: R ranks, S tokens per rank, K experts per token (top-K), E experts,
 * E_R = E/R experts homed contiguously per rank (expert e lives on rank
 * floor(e/E_R)), H hidden size, T = R*S tokens, P = T*K routed (token, k)
 * pairs, flattened pair index p = t*K + k.  The dispatch buffer has P rows; rank
 * r owns rows [r*S*K, (r+1)*S*K).
 *
 * Conventions shared by every call:
 *  - Array arguments are DEVICE pointers, owned by the caller, unless a comment
 *    says "host".  Bases must be 16-byte aligned; row-major, contiguous.
 *  - bf16 data are passed as uint16_t bit patterns.
 *  - Every call that takes a stream only enqueues work on it: no host
 *    synchronisation, no device or host allocation.  ep_status_read is the one
 *    call that waits.
 *  - Return value: EP_OK, or a negative EP_ERR_* code when an argument is
 *    invalid (nothing is enqueued) or a launch failed.
 *  - Problems the device detects (an expert id outside [0, E), a row index
 *    outside the buffer, loads that do not add up, a bounded wait that ran out)
 *    are OR-ed as EP_DEV_* bits into the caller's int32 *dev_status; the outputs
 *    are then defined but unspecified, and no write goes out of bounds.
 *  - Limits: 1 <= K <= min(E, 32), E <= EP_MAX_EXPERTS, R <= EP_MAX_RANKS,
 *    E % R == 0, H % 8 == 0, P < 2^31.
 *  - The row movers (dispatch; combine, which also serves as the backward of
 *    dispatch; the replica gradient reduction; one-buffer and rank-local
 *    forms) are launched with programmatic dependent launch: the GPU may
 *    schedule them while the preceding kernel in the stream finishes, and
 *    each waits for that kernel's completion before touching memory, so
 *    stream order holds as for any launch.
 *  - A workspace (ws) holds the counters and grid-barrier words of the call
 *    that uses it: calls in flight at the same time (on different streams)
 *    need workspaces of their own.  Calls on one stream may share one.
 *  - The dispatch buffer and the combine input are views that the next dispatch
 *    or combine overwrites ([GR] "Ένα ρεαλιστικό πλαίσιο αξιολόγησης πριν από
 *    την υιοθέτηση": zero-copy views must not be kept past the next dispatch or
 *    combine, nor saved by autograd).
 */
#ifndef TDH_EP_H
#define TDH_EP_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define EP_OK 0
#define EP_ERR_ARG (-1)      /* invalid argument; nothing enqueued */
#define EP_ERR_CAPACITY (-2) /* a caller buffer is too small; nothing enqueued */
#define EP_ERR_CUDA (-3)     /* a CUDA launch or copy failed */

#define EP_DEV_BAD_EXPERT_ID 0x1     /* a topk id outside [0, E) */
#define EP_DEV_LOOKBACK_TIMEOUT 0x2  /* a bounded inter-block wait gave up */
#define EP_DEV_BAD_LOADS 0x4         /* loads do not sum to R*S*K, or are negative */
#define EP_DEV_BAD_ROW 0x8           /* a row index outside the buffer */
#define EP_DEV_COPY_TIMEOUT 0x10     /* a bounded wait on an asynchronous copy gave up */

#define EP_MAX_EXPERTS 1024
#define EP_MAX_RANKS 1024

#define EP_DTYPE_F32 0
#define EP_DTYPE_BF16 1

/*
 * Layout of the plan buffer (int32 words) written by ep_plan.  Every field is an
 * offset, in int32 elements, from the start of the buffer; `words` is its size.
 * cap = E + R - 1 bounds the number of replicas (each replica ends at a chunk
 * boundary or a deficit boundary: at most E chunks plus R deficits, minus one).
 * Slot ids: e for the home copy of expert e, E + m for replica m.
 */
typedef struct {
  int64_t words;      /* total size in int32 elements */
  int32_t cap;        /* E + R - 1 */
  int32_t n_rep;      /* [1] number of replicas */
  int32_t n_chunks;   /* [1] number of replicated experts (chunks) */
  int32_t rank_load;  /* [R] L_r = sum of T_e over rank r's home experts */
  int32_t rank_nrep;  /* [R] replicas received by rank r */
  int32_t rank_rep_first; /* [R] match index of rank r's first received replica
                             (= replicas received by ranks < r) */
  int32_t home_count; /* [E] pairs kept by the home copy of e */
  int32_t home_base;  /* [E] first buffer row of the home copy of e */
  int32_t copy_first; /* [E] match index of e's first replica (0 if none) */
  int32_t copy_cnt;   /* [E] number of replicas of e */
  int32_t rep_expert; /* [cap] logical expert of replica m (match order) */
  int32_t rep_rank;   /* [cap] receiving rank of replica m */
  int32_t rep_count;  /* [cap] pairs taken by replica m */
  int32_t rep_begin;  /* [cap] offset of replica m's range in e's pair list */
  int32_t rep_base;   /* [cap] first buffer row of replica m */
  int32_t rep_experts;/* [E] replicated experts in match order (n_chunks valid) */
  int32_t slot_order; /* [E + cap] slot ids in buffer order; -1 past E + n_rep */
  int32_t cu_seqlens; /* [E + cap + 1] first row of each slot in buffer order;
                         entries from E + n_rep on hold R*S*K */
} EpPlanLayout;

/*
 * Layout of the quota-plan buffer written by ep_quota_route: offsets in int32
 * elements into one int32 array, each region 32-byte aligned.  Instance i of
 * the plan is the home copy of expert i for i < E and replica i - E after.
 */
typedef struct {
  int64_t words;          /* total size in int32 elements */
  int32_t cap;            /* E + R - 1 */
  int32_t tau;            /* [1] tau*, the rank-load threshold met (-1: no plan) */
  int32_t n_rep;          /* [1] number of replicas */
  int32_t n_local;        /* [1] pairs placed on their own source rank */
  int32_t n_chunks;       /* [1] number of replicated experts */
  int32_t rank_load;      /* [R] rows of rank r (<= tau) */
  int32_t rank_off;       /* [R] first buffer row of rank r */
  int32_t rank_nrep;      /* [R] replicas received by rank r */
  int32_t rank_rep_first; /* [R] replicas received by ranks < r */
  int32_t home_quota;     /* [E] pairs taken by the home copy of e */
  int32_t rep_first;      /* [E] match index of e's first replica (0 if none) */
  int32_t rep_cnt;        /* [E] number of replicas of e */
  int32_t rep_experts;    /* [E] replicated experts in match order (n_chunks valid, -1 after) */
  int32_t rep_expert;     /* [cap] logical expert of replica m (match order) */
  int32_t rep_rank;       /* [cap] receiving rank of replica m */
  int32_t rep_count;      /* [cap] quota of replica m */
  int32_t inst_local;     /* [E + cap] local pairs of instance i: min(quota, L[rank][e]) */
  int32_t inst_cum;       /* [E + cap] looked-up pairs of e's earlier instances */
  int32_t inst_base;      /* [E + cap] first buffer row of instance i */
  int32_t inst_lpre;      /* [E + cap] pairs of e from source ranks below instance i's rank */
  int32_t rep_local_incl; /* [cap] local pairs of e's replicas up to and including m */
  int32_t slot_order;     /* [E + cap] instance ids in buffer order; -1 past E + n_rep */
  int32_t cu_seqlens;     /* [E + cap + 1] first row of each slot in buffer order;
                             entries from E + n_rep on hold R*S*K */
} EpQuotaLayout;

/* Library version string (host). */
EP_API const char* ep_version(void);

/* Number of CUDA kernels this library has launched in this process (host
 * counter, incremented at each launch). */
EP_API uint64_t ep_launch_count(void);

/*
 * Bytes of scratch (`ws`) that ep_route_stats, ep_layout and ep_align_sort need
 * for T tokens, K, E.  Host only.  The same ws must be passed to ep_route_stats
 * and then ep_layout for the same topk_ids: ep_layout reads the per-tile
 * per-expert prefix counts that ep_route_stats left there.
 */
EP_API int ep_workspace_size(int64_t T, int K, int E, size_t* bytes /* host out */);

/* Fill *layout (host) with the plan buffer layout for E, R.  Host only. */
EP_API int ep_plan_layout(int E, int R, EpPlanLayout* layout /* host out */);

/*
 * a1. Per-expert loads and imbalance.  [FR] "Pourquoi le parallélisme d'experts
 * est-il nécessaire": max_vio = max_e(T_e / T̄) - 1, 0 for perfect balance;
 * T̄ is the mean load P/E.
 *   topk_ids [T, K] int32: expert of pair p = t*K + k.
 *   loads    [E] int32 out: T_e = #{p : topk_ids[p] == e}.
 *   max_vio  [1] double out: (max_e T_e) * E / P - 1 in fp64 (0 when P == 0).
 *   ws       scratch of ep_workspace_size bytes; keeps per-tile prefix counts.
 * One histogram pass with a single-pass decoupled look-back scan over tiles;
 * integer adds only, so the result does not depend on scheduling.
 */
EP_API int ep_route_stats(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads, double* max_vio, void* ws,
                   size_t ws_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * a2. Replica plan.  [GR] "Η βασική υπόσχεση του MoonEP: σταθερό φορτίο S × K":
 * every rank ends with exactly S*K pairs, by copying hot experts to other ranks
 * for this step.  Rule (the pages leave it open; this library's deterministic
 * reading): rank load L_r; an overloaded rank's excess L_r - S*K is cut into
 * chunks taken from its home experts in descending id (chunk = min(T_e, excess
 * left)); underloaded ranks' deficits S*K - L_r are taken in ascending rank;
 * the two sequences are matched by a merge over their prefix sums, and every
 * piece of the merge is one replica (expert, receiving rank, count), in "match
 * order".
 *   loads [E] int32 (from ep_route_stats); must sum to R*S*K.
 *   plan  int32 buffer of EpPlanLayout.words elements, written in full.
 * One block of 1024 threads.
 */
EP_API int ep_plan(const int32_t* loads, int R, int64_t S, int K, int E, int32_t* plan, size_t plan_words,
            int32_t* dev_status, cudaStream_t stream);

/*
 * Quota-driven replica planning with a per-rank replica budget.  [JA]
 * "その仕組みは高速なエキスパート複製に依存する" (remio.ai UltraEP article):
 * from the exact load matrix after routing (pairs of each source rank per
 * expert), a load threshold is searched for that every rank can stay under
 * within the replica slots available; the planner decides which heavy experts
 * get copies, on which ranks, and how many pairs each instance takes; copies
 * exist only with work; pairs use a local instance first and the rest of the
 * demand is placed by lookup on cumulative quotas; all on the GPU.
 * Rule (this library's reading; the page prints none):
 *   - source rank of pair p = p / (S*K); home rank of e = e / (E/R); H_r = the
 *     loads of rank r's home experts;
 *   - at threshold tau, rank r sheds max(0, H_r - tau) pairs from its home
 *     experts heaviest first (ties: lower id), each chunk = min(T_e, excess
 *     left); ranks with H_r < tau take pieces in ascending rank order (one
 *     replica per piece) until full or holding B pieces; tau is feasible when
 *     every chunk is placed;
 *   - tau* = the smallest feasible tau from ceil(P/R) up (max H_r always is);
 *   - instances of e: home, then its replicas in match order.  Instance i on
 *     rank r_i takes the first min(q_i, L[r_i][e]) pairs of e from source rank
 *     r_i; the other pairs of e, in pair order, fill the instances' remaining
 *     quotas in instance order;
 *   - rows: rank after rank (rank r holds rank_load[r] <= tau* rows); within a
 *     rank home experts by id then received replicas by match order; within an
 *     instance its local pairs then its looked-up pairs, each in pair order.
 * Arguments:
 *   topk_ids [T, K] int32 device, T = R*S.
 *   B        replicas a rank may hold (>= 0).
 *   loads    [E] int32 device out: T_e.
 *   plan     int32 device out, layout from ep_quota_plan_layout.
 *   pos, src [T*K] int32 device out: row of each pair, pair of each row.
 *   ws       device scratch of ep_quota_workspace_size bytes (contents need
 *            not be initialised).
 * Four launches (rank-aligned tile histogram, column scan, threshold search
 * over all candidates at once, stable-rank walk); integer work only, so the
 * result does not depend on scheduling.  EP_ERR_ARG for bad shapes (E % R,
 * K > E, ...) or B < 0; EP_ERR_CAPACITY when plan_words or ws_bytes is short.
 * Expert ids outside [0, E) set EP_DEV_BAD_EXPERT_ID and leave tau = -1 and
 * pos = -1.
 */
EP_API int ep_quota_workspace_size(int64_t T, int K, int E, int R, size_t* bytes /* host out */);
EP_API int ep_quota_plan_layout(int E, int R, EpQuotaLayout* layout /* host out */);
EP_API int ep_quota_route(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int B, int32_t* loads,
                          int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src, void* ws, size_t ws_bytes,
                          int32_t* dev_status, cudaStream_t stream);

/*
 * ep_replica_grad_reduce for a plan from ep_quota_route: the same reduction
 * (g_home[e] += each replica's row of e in match order, fp32), the replica
 * list read from the quota plan.  Arguments as in ep_replica_grad_reduce;
 * g_rep has at least n_rep rows.
 */
EP_API int ep_quota_replica_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, int R,
                                        const int32_t* plan, size_t plan_words, int clear_replicas,
                                        int32_t* dev_status, cudaStream_t stream);

/*
 * Prefetch slots under a per-rank budget B.  [GR] "Το memory contract που
 * πρέπει να καταλάβει η τεχνική ομάδα": each rank's grouped-GEMM weights are
 * [E+B, H, H'], rows E..E+B-1 being local prefetch slots, and replicas beyond
 * the slots read their weights from the home rank (B = E/R for training, 3-4
 * for inference).  The j-th replica a rank receives, in match order, gets
 * weight row E + j while j < B, else -1; the token layout is unchanged.
 *   plan         from ep_plan (device).
 *   SK           S*K, the pairs per rank.
 *   slot         [cap] int32 out (device; -1 past n_rep too).
 *   n_remote     [R] int32 out (device): replicas rank r reads from home.
 *   load_capped  [R] int64 out (device) or NULL: the other reading of the
 *                overflow, where a replica without a slot is not made and its
 *                pairs stay with the expert's home rank; rank r's load is then
 *                S*K - (pairs of its slotless replicas) + (pairs of slotless
 *                replicas of its own experts).
 * One launch, nothing allocated.  EP_ERR_ARG for a bad shape, B < 0 or a
 * NULL required pointer; EP_ERR_CAPACITY when plan_words is short.
 */
EP_API int ep_prefetch_slots(const int32_t* plan, size_t plan_words, int E, int R, int64_t SK, int B,
                             int32_t* slot, int32_t* n_remote, int64_t* load_capped, cudaStream_t stream);

/*
 * a3. Layout.  [GR] "Online planning, zero copy και στατικά σχήματα": each pair
 * goes straight to its final row, grouped by expert, in a static S*K buffer per
 * rank.  Stable counting sort by expert, ties in flattened (rank, token, k)
 * order; the home copy takes an expert's first home_count pairs, its replicas
 * the following ranges in match order; rank r's rows hold its home experts in
 * id order, then its received replicas in match order.
 *   pos       [P] int32 out: row of pair p.
 *   src       [P] int32 out: pair of row i (inverse of pos).
 *   pair_slot [P] int32 out, may be NULL: slot id of pair p (e or E + m).
 *   plan      from ep_plan for the loads of these topk_ids.
 *   ws        the scratch ep_route_stats filled for these topk_ids.
 */
EP_API int ep_layout(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, const int32_t* plan,
              size_t plan_words, const void* ws, size_t ws_bytes, int32_t* pos, int32_t* src, int32_t* pair_slot,
              int32_t* dev_status, cudaStream_t stream);

/*
 * a4. MoE Align & Sort.  [ZH]: sort the routed ids by expert and pad each
 * expert's group to a multiple of block_m so every block of the grouped GEMM
 * belongs to one expert.  Readings: the ids are flattened pair indices p
 * (token = p / K), stable in p; padding holds the sentinel P.
 *   sorted_token_ids [sorted_cap] int32 out, sorted_cap >= P + E*(block_m-1):
 *       group of e at off_e = sum_{e'<e} ceil(c_e'/block_m)*block_m, then P
 *       as padding up to the next multiple of block_m, and P past the end.
 *   expert_ids [expert_ids_cap] int32 out, >= ceil(sorted_cap / block_m):
 *       expert of each block, -1 past num_tokens_post_pad / block_m.
 *   num_tokens_post_pad [1] int32 out: sum_e ceil(c_e/block_m)*block_m.
 *   ws  scratch of ep_workspace_size bytes (its histogram is rebuilt here).
 */
EP_API int ep_align_sort(const int32_t* topk_ids, int64_t T, int K, int E, int block_m, int32_t* sorted_token_ids,
                  int64_t sorted_cap, int32_t* expert_ids, int64_t expert_ids_cap, int32_t* num_tokens_post_pad,
                  void* ws, size_t ws_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * a1-a4 in one launch: the outputs of ep_route_stats, ep_plan, ep_layout and
 * (when sorted_token_ids is not NULL) ep_align_sort, bit for bit, from one
 * cooperative kernel whose CTAs meet at grid barriers (all waits bounded).
 * The route phase moves only a few bytes per pair, so it is latency-bound; one
 * resident grid replaces four launches and the serial look-back.  When the
 * grid cannot be co-resident it runs the four separate calls instead.
 * Arguments as in those calls; ws is ep_workspace_size bytes (its contents
 * afterwards are not the per-tile prefixes ep_layout reads).
 */
EP_API int ep_route_fused(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S, int32_t* loads,
                          double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos, int32_t* src,
                          int32_t* pair_slot, int block_m, int32_t* sorted_token_ids, int64_t sorted_cap,
                          int32_t* expert_ids, int64_t expert_ids_cap, int32_t* num_tokens_post_pad, void* ws,
                          size_t ws_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * Fused layout + dispatch: ep_route_fused followed by ep_dispatch(x, T, K, H,
 * pos, buf, buf_rows) in one cooperative launch, same outputs bit for bit
 * (every route output, and buf[pos[p]] = x[p / K] for every pair).  [GR]
 * "Online planning, zero copy και στατικά σχήματα": the rows go straight to
 * their final expert-grouped position; here each tile CTA copies the token
 * rows of its own pairs as soon as it has placed them, with no launch or
 * grid-wide wait between layout and dispatch.  Token rows whose pairs fall in
 * two tiles are read twice (at most one extra row per tile).
 *   x    [T, H] bf16 in (non-NULL when T > 0), buf [buf_rows, H] bf16 out, H as in
 *        ep_dispatch (H % 8 == 0, 8 <= H, 2H <= 1 MiB); both 16-byte aligned.
 * Other arguments as in ep_route_fused.  When the grid with its row stages
 * cannot be co-resident it runs ep_route_fused's fallback and ep_dispatch.
 * Errors: as ep_route_fused and ep_dispatch (EP_DEV_BAD_ROW for a pair whose
 * row is outside the buffer, EP_DEV_COPY_TIMEOUT for a copy that did not land).
 */
EP_API int ep_route_dispatch_fused(const int32_t* topk_ids, int64_t T, int K, int E, int R, int64_t S,
                                   int32_t* loads, double* max_vio, int32_t* plan, size_t plan_words, int32_t* pos,
                                   int32_t* src, int32_t* pair_slot, int block_m, int32_t* sorted_token_ids,
                                   int64_t sorted_cap, int32_t* expert_ids, int64_t expert_ids_cap,
                                   int32_t* num_tokens_post_pad, const uint16_t* x, int64_t H, uint16_t* buf,
                                   int64_t buf_rows, void* ws, size_t ws_bytes, int32_t* dev_status,
                                   cudaStream_t stream);

/*
 * a5. Dispatch.  [GR] "Online planning, zero copy και στατικά σχήματα": rows are
 * written in place into the expert-grouped buffer, no intermediate copy.
 *   x   [T, H] bf16; buf [buf_rows, H] bf16 out; buf[pos[p]] = x[p / K] bitwise.
 *   Rows whose pos is outside [0, buf_rows) are skipped and flagged.
 *   Rows up to about 100 KB (two shared-memory stages of one row each within
 *   200 KB: H <= 51,136 at K <= 8); wider rows get EP_ERR_ARG.
 * Each token row is read once (TMA bulk copy into shared memory) and written to
 * its K rows by bulk stores.
 */
EP_API int ep_dispatch(const uint16_t* x, int64_t T, int K, int64_t H, const int32_t* pos, uint16_t* buf,
                int64_t buf_rows, int32_t* dev_status, cudaStream_t stream);

/*
 * Stand-in for the expert computation (the grouped GEMM is outside this
 * library's path), for tests and examples: y[i] = bf16_rn(float(buf[i]) *
 * scale[e]) with e = topk_ids[src[i]], fp32 multiply.  y may alias buf.
 */
EP_API int ep_expert_scale(const uint16_t* buf, int64_t rows, int64_t H, const int32_t* src, const int32_t* topk_ids,
                    int64_t P, const float* scale, int E, uint16_t* y, int32_t* dev_status, cudaStream_t stream);

/*
 * a6. Combine.  out[t] = bf16_rn( sum_{k=0..K-1} w[t,k] * float(y[pos[t*K+k]]) ),
 * accumulated in fp32 in k order from 0, each product and sum rounded
 * separately (no fused multiply-add), one rounding to bf16 at the end.
 *   y [y_rows, H] bf16; w [T, K] fp32 (NULL: unit weights); pos [P] int32; out [T, H] bf16 out.
 *   Pairs whose pos is outside [0, y_rows) contribute nothing and are flagged.
 *   From T*H >= 2^28 with K <= 8 the rows are read through a per-warp
 *   shared-memory ring (cp.async); below, each thread loads its K vectors into
 *   registers.  The two give the same bits.
 */
EP_API int ep_combine(const uint16_t* y, int64_t y_rows, const float* w, const int32_t* pos, int64_t T, int K, int64_t H,
               uint16_t* out, int32_t* dev_status, cudaStream_t stream);

/*
 * Backward of dispatch: the MoE Align & Sort report [ZH] recalls that the
 * permute recording the source -> destination mapping has unpermute as its
 * gradient.  dx[t] = bf16_rn( sum_{k} float(dbuf[pos[t*K+k]]) ), fp32 in k
 * order, one rounding (combine with unit weights).
 *   dbuf [buf_rows, H] bf16 (gradient w.r.t. the dispatched rows); dx [T, H] out.
 */
EP_API int ep_dispatch_backward(const uint16_t* dbuf, int64_t buf_rows, const int32_t* pos, int64_t T, int K,
                                int64_t H, uint16_t* dx, int32_t* dev_status, cudaStream_t stream);

/*
 * Backward of combine, given dout [T, H] bf16 (gradient w.r.t. out):
 *   dy[pos[t*K+k]] = bf16_rn(w[t,k] * float(dout[t]))   (gradient w.r.t. the expert rows)
 *   dw[t,k] = sum_h float(dout[t,h]) * float(y[pos[t*K+k], h])   fp32, summation
 *             order unspecified (within H * 2^-24 * sum|dout*y| of the exact value)
 *   y [y_rows, H] bf16 (combine's input); dy [y_rows, H] out (rows no pair
 *   addresses are left untouched); dw [T, K] fp32 out; 1 <= K <= 8.
 * Each dout row is read once, each y row once, each dy row written once.
 */
EP_API int ep_combine_backward(const uint16_t* dout, const float* w, const uint16_t* y, int64_t y_rows,
                               const int32_t* pos, int64_t T, int K, int64_t H, uint16_t* dy, float* dw,
                               int32_t* dev_status, cudaStream_t stream);

/*
 * a7. Replica gradient reduction.  [GR] "Τι συμβαίνει στους gradients κατά την
 * εκπαίδευση": replica gradients live in a separate reduce buffer in fp32 and
 * are added into the home expert's gradient, after which the used slots are
 * cleared.  Per element: g_home[e] = ((g_home[e] + g_rep[m1]) + g_rep[m2]) ...
 * over e's replicas in match order, fp32, one add at a time.
 *   g_home [E, n] fp32 in/out.  g_rep [cap, n], row m = replica m, fp32
 *   (EP_DTYPE_F32) or bf16 (EP_DTYPE_BF16, widened exactly).
 *   clear_replicas != 0 zeroes the rows of the replicas used.
 */
EP_API int ep_replica_grad_reduce(float* g_home, const void* g_rep, int rep_dtype, int64_t n, int E, int R,
                           const int32_t* plan, size_t plan_words, int clear_replicas, int32_t* dev_status,
                           cudaStream_t stream);

/*
 * ---------------------------------------------------------------------------
 * Rank-local form: the calls one rank makes when the R ranks are R processes
 * (one GPU each) rather than R partitions of one buffer.  [GR] "Online
 * planning, zero copy και στατικά σχήματα": tokens are written straight into
 * their final expert-grouped rows on the remote ranks, and the application
 * reads views of that communication buffer.  [JA] "その仕組みは高速な
 * エキスパート複製に依存する": planning starts from the exact source-rank x
 * expert load matrix after routing.  Flow on rank r:
 *   1. ep_route_stats(topk_local [S, K], T = S) -> counts row r (its pairs per
 *      expert) and, in ws, the per-tile prefixes ep_layout_rank reads;
 *   2. the caller all-gathers the rows into counts [R, E] (one collective);
 *   3. ep_plan_from_counts: the same plan on every rank, no further exchange;
 *   4. ep_layout_rank: the global row of each local pair; a pair's rank in its
 *      expert's list is (pairs of that expert on source ranks < r) + (its rank
 *      among the local pairs), so no other coordination is needed;
 *   5. ep_dispatch_peer / ep_combine_peer / ep_replica_grad_reduce_peer move
 *      rows through a table of the R ranks' buffer base addresses.
 * Every output equals, bit for bit, the slice of the one-buffer path's output
 * that belongs to rank r.  Peer tables: device arrays of R uint64 device
 * addresses (this GPU's own buffer or peers' buffers mapped into its address
 * space, e.g. symmetric memory or IPC); each must be 16-byte aligned.  Rows:
 * pos_local holds global rows g in [0, total_rows).  With rank_first_row NULL
 * every rank holds rows_per_rank rows and g lives on rank g / rows_per_rank
 * (the exact-S*K plan: rows_per_rank = S*K); otherwise rank d's rows start at
 * rank_first_row[d] (device int32 [R], ascending, from 0; a quota plan's
 * rank_off) and its buffer holds rows_per_rank rows.  A zero or misaligned
 * table entry, or a row past its rank's buffer, is never dereferenced: the
 * rows it would serve are skipped and EP_DEV_BAD_ROW is set.
 */

/*
 * Peer buffers across processes (host calls, no stream; set-up, not part of a
 * step).  [GR] "Online planning, zero copy και στατικά σχήματα": a sending rank
 * writes rows straight into the receiving rank's buffer, so that buffer must
 * be mapped into the sender's address space.  With one process per rank this
 * is done with CUDA IPC handles:
 *   ep_ipc_export: dev_ptr (device, a buffer from cudaMalloc or a caching
 *     allocator built on it; not VMM/cuMemMap memory) -> *handle (host,
 *     EP_IPC_HANDLE_BYTES opaque bytes naming the allocation that holds
 *     dev_ptr) and *offset (host, dev_ptr's byte offset in that allocation).
 *   ep_ipc_open (in another process): *base = the allocation mapped here,
 *     *dev_ptr = *base + offset, usable in a peer table.  Opening a handle
 *     exported by the same process fails (EP_ERR_CUDA): a rank uses its own
 *     pointer for itself.  Peer access to another GPU is enabled by the driver.
 *   ep_ipc_close(base): unmaps (every process that opened a handle closes it
 *     before the owner frees the buffer).
 * Returns EP_OK, EP_ERR_ARG (null argument, or dev_ptr not device memory) or
 * EP_ERR_CUDA.  The handles carry no synchronisation: the caller orders the
 * ranks' kernels (e.g. every rank's dispatch done before any rank's combine).
 */
#define EP_IPC_HANDLE_BYTES 64
EP_API int ep_ipc_export(const void* dev_ptr, void* handle /* host out */, uint64_t* offset /* host out */);
EP_API int ep_ipc_open(const void* handle /* host */, uint64_t offset, void** base /* host out */,
                       void** dev_ptr /* host out */);
EP_API int ep_ipc_close(void* base);

/*
 * The plan from the gathered load matrix: loads[e] = sum_r counts[r, e], then
 * exactly ep_plan.  counts [R, E] int32 device; loads [E] int32 out (device) or
 * NULL; plan as in ep_plan.  One CTA.
 */
EP_API int ep_plan_from_counts(const int32_t* counts, int R, int64_t S, int K, int E, int32_t* loads, int32_t* plan,
                               size_t plan_words, int32_t* dev_status, cudaStream_t stream);

/*
 * Rows of rank `rank`'s own pairs.  topk_local [S, K] int32; counts [R, E] from
 * step 2; plan from ep_plan_from_counts; ws the scratch ep_route_stats filled
 * for topk_local (T = S).  pos_local [S*K] int32 out: the global row of local
 * pair i (= pos[rank*S*K + i] of the one-buffer layout).  pair_slot [S*K] out
 * or NULL.  No src output: a receiving rank finds a row's expert from the plan's
 * slot table (cu_seqlens, slot_order).
 */
EP_API int ep_layout_rank(const int32_t* topk_local, int64_t S, int K, int E, int R, int rank,
                          const int32_t* counts, const int32_t* plan, size_t plan_words, const void* ws,
                          size_t ws_bytes, int32_t* pos_local, int32_t* pair_slot, int32_t* dev_status,
                          cudaStream_t stream);

/*
 * Dispatch of rank-local tokens: the row of x_local [S, H] bf16 of pair i goes
 * to global row pos_local[i] in the rank buffers (H bf16 per row).  One TMA
 * bulk load per token row and K bulk stores, as ep_dispatch.
 */
EP_API int ep_dispatch_peer(const uint16_t* x_local, int64_t S, int K, int64_t H, const int32_t* pos_local,
                            const uint64_t* peer_bufs, const int32_t* rank_first_row, int R, int64_t rows_per_rank,
                            int64_t total_rows, int32_t* dev_status, cudaStream_t stream);

/*
 * Combine of rank-local tokens, reading the expert rows from the R rank
 * buffers: out_local[t] = bf16_rn( sum_k w_local[t,k] * float(row pos_local[t*K+k]) ),
 * fp32 in k order, as ep_combine.  w_local NULL: unit weights (the backward of
 * dispatch, as ep_dispatch_backward).  1 <= K <= 8.
 */
EP_API int ep_combine_peer(const uint64_t* peer_bufs, const int32_t* rank_first_row, int R, int64_t rows_per_rank,
                           int64_t total_rows, const float* w_local, const int32_t* pos_local, int64_t S, int K,
                           int64_t H, uint16_t* out_local, int32_t* dev_status, cudaStream_t stream);

/*
 * Replica gradient reduction on the home rank.  [GR] "Τι συμβαίνει στους
 * gradients κατά την εκπαίδευση": each rank views the R ranks' reduce buffers
 * together and reads, over NVLink, the slots that hold its own experts'
 * replica gradients, adds them into its local parameter gradient and clears
 * the used slots.  Per element of each home expert e of `rank` with replicas:
 *   g_home_local[e - rank*E/R] = ((g + rep(m1)) + rep(m2)) ...  (match order, fp32)
 * where replica m's row is row (m - first replica rank d receives) of rank d's
 * reduce buffer, d = the replica's receiving rank: the replicas a rank receives
 * are consecutive in match order.
 *   g_home_local [E/R, n] fp32 in/out; peer_g_rep: device table of R addresses
 *   of [rep_rows, n] reduce buffers (fp32 or bf16 by rep_dtype), row j = the
 *   j-th replica that rank receives; a replica with j >= rep_rows (no row) is
 *   skipped and flagged EP_DEV_BAD_ROW (a rank receives at most E - E/R
 *   replicas under any plan);
 *   plan from ep_plan_from_counts; clear_replicas != 0 zeroes the rows used.
 */
EP_API int ep_replica_grad_reduce_peer(float* g_home_local, const uint64_t* peer_g_rep, int64_t rep_rows,
                                       int rep_dtype, int64_t n, int E, int R, int rank, const int32_t* plan,
                                       size_t plan_words, int clear_replicas, int32_t* dev_status,
                                       cudaStream_t stream);

/*
 * The quota-driven planner (ep_quota_route) in rank-local form.  Flow on rank
 * r: ep_route_stats(topk_local) -> counts row and per-tile prefixes in ws; the
 * all-gather of the rows into counts [R, E] (exactly the source-rank x expert
 * load matrix the planner starts from); ep_quota_plan_from_counts (the same
 * plan on every rank); ep_quota_layout_rank (global rows of the rank's own
 * pairs).  Then ep_dispatch_peer / ep_combine_peer with rank_first_row = the
 * plan's rank_off array (rank r holds rank_load[r] <= tau* rows, so a buffer of
 * rows_per_rank >= tau* rows per rank suffices; tau* <= max(ceil(P/R), max_r
 * of the rank's home loads)), and ep_quota_replica_grad_reduce_peer.
 */
EP_API int ep_quota_counts_workspace_size(int E, int R, size_t* bytes /* host out */);

/*
 * counts [R, E] int32 device (gathered); loads [E] int32 out (T_e); plan as in
 * ep_quota_route (EpQuotaLayout); ws device scratch of
 * ep_quota_counts_workspace_size bytes.  Two launches.  Counts that do not add
 * up to R*S*K (or are negative) give tau = -1 and no replica.
 */
EP_API int ep_quota_plan_from_counts(const int32_t* counts, int R, int64_t S, int K, int E, int B, int32_t* loads,
                                     int32_t* plan, size_t plan_words, void* ws, size_t ws_bytes,
                                     int32_t* dev_status, cudaStream_t stream);

/*
 * Rows of rank `rank`'s own pairs under a quota plan: pos_local[i] = pos[rank*S*K
 * + i] of ep_quota_route for the whole problem.  ws is the scratch
 * ep_route_stats filled for topk_local (T = S); counts the gathered matrix.
 */
EP_API int ep_quota_layout_rank(const int32_t* topk_local, int64_t S, int K, int E, int R, int rank,
                                const int32_t* counts, const int32_t* plan, size_t plan_words, const void* ws,
                                size_t ws_bytes, int32_t* pos_local, int32_t* dev_status, cudaStream_t stream);

/* ep_replica_grad_reduce_peer for a plan from ep_quota_plan_from_counts. */
EP_API int ep_quota_replica_grad_reduce_peer(float* g_home_local, const uint64_t* peer_g_rep, int64_t rep_rows,
                                             int rep_dtype, int64_t n, int E, int R, int rank, const int32_t* plan,
                                             size_t plan_words, int clear_replicas, int32_t* dev_status,
                                             cudaStream_t stream);

/*
 * ep_route_stats without a scratch argument, for callers that cannot allocate
 * device memory for it: hosts that pass a kernel only its inputs and outputs at
 * enqueue time and forbid allocation there, or runtimes whose device memory is
 * all planned in advance.  The source pages have no counterpart of this call;
 * it computes the same loads and max_vio as ep_route_stats, bit for bit.
 *   Scratch: a fixed array of EP_NOALLOC_SCRATCH_BYTES inside the library,
 *   present on every GPU that loads it until the process exits.  The problem
 *   must fit: about 12 * ceil(T*K / tile) * E + 4*E + 512 bytes, tile = 2048,
 *   4096 or 8192 pairs (as ep_workspace_size reports for the same T, K, E);
 *   larger problems get EP_ERR_CAPACITY and nothing is enqueued.
 *   The first call in a CUDA context (with that context's device current)
 *   looks the array's device address up with cudaGetSymbolAddress and caches
 *   it with the context's unique id; a later call under a different context of
 *   the same device (after cudaDeviceReset, or a context the caller created)
 *   looks it up again.  Make the first call in each context before any stream
 *   capture.  No call allocates (no cudaMalloc, cudaFree or allocating library
 *   routine).
 *   All calls share the one array and it keeps the previous call's contents:
 *   calls whose work overlaps on the GPU (other streams, other threads) race
 *   on it and must be serialised by the caller.  ep_layout cannot use this
 *   call's per-tile counts; use ep_route_stats with a workspace for that.
 */
#define EP_NOALLOC_SCRATCH_BYTES (4u << 20)
EP_API int ep_route_stats_noalloc(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads, double* max_vio,
                                  int32_t* dev_status, cudaStream_t stream);

/*
 * Self-test of failure detection (no counterpart on the pages): runs
 * ep_route_stats' kernel with its first tile never scheduled, so every other
 * tile's look-back waits on a flag that nothing sets.  The waits run out after
 * about one second, EP_DEV_LOOKBACK_TIMEOUT is OR-ed into *dev_status, and the
 * CUDA context stays usable.  Needs T*K above one tile (> 2048 pairs).  Waits
 * for the stream before returning.  loads and max_vio come out wrong by design.
 */
EP_API int ep_selftest_lookback_timeout(const int32_t* topk_ids, int64_t T, int K, int E, int32_t* loads,
                                        double* max_vio, void* ws, size_t ws_bytes, int32_t* dev_status,
                                        cudaStream_t stream);

/* Copy *dev_status to *host_status (host) after the work queued on `stream`;
 * waits for the stream.  The only synchronising call. */
EP_API int ep_status_read(const int32_t* dev_status, int32_t* host_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TDH_EP_H */
