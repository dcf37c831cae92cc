/*
 * CPU ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded C restatement of what the expert-parallel
 * dispatch path computes, written from the source pages' definitions.  Only the
 * test suite, the package's smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only in the seeded inputs of the workload module.
 *
 * Sources (cited by page title and section):
 *  [GR] "MoonEP: πώς η εξισορρόπηση των AI experts αλλάζει την υποδομή των
 *       MoE μοντέλων" (twodots.gr)
 *  [FR] "Moonshot AI открыла код MoonEP — библиотеки для обучения MoE-модели
 *       Kimi K3" (news.hamidun.com)
 *  [ZH] the MoE Align & Sort report (新智元报道, los70adestajo.com page)
 *  [JA] "Xiaohongshuと北京大学がUltraEPを発表、静的MoE負荷分散に挑戦" (remio.ai)
 *
 * Notation: R ranks, S tokens per rank, K experts per token, E experts,
 * E_R = E/R experts homed per rank, T = R*S tokens, P = T*K routed pairs,
 * flattened pair index p = t*K + k.  Rank r owns buffer rows [r*S*K, (r+1)*S*K).
 *
 * Floating point: the pages fix fp32 accumulation for combine and gradient
 * reduction and bf16 rows, so those are done in fp32 here, one IEEE operation
 * at a time (the file is compiled with -ffp-contract=off: no fused multiply-add).
 * max_vio is computed in fp64.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bf16 */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* round to nearest, ties to even; NaN stays NaN */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------ 1. stats */
/*
 * [FR] "Pourquoi le parallélisme d'experts est-il nécessaire": the imbalance
 * metric is max_vio = max_e(T_e / T̄) - 1, zero meaning perfect balance; [GR]
 * "Γιατί τα Mixture-of-Experts δημιουργούν πρόβλημα κατανομής" says the same.
 * T_e = number of routed (token, k) pairs whose expert is e.  T̄ is read as
 * the mean of T_e over the E experts, P / E, the only choice for which a
 * perfectly even routing gives 0.  max_e(T_e / (P/E)) - 1 is evaluated as
 * (max_e T_e) * E / P - 1 in fp64 (the product is exact).
 *
 * Returns the number of ids outside [0, E); those pairs are not counted.
 */
int64_t oracle_route_stats(const int32_t* topk, int64_t T, int K, int E, int32_t* loads, double* max_vio) {
  int64_t P = T * (int64_t)K, bad = 0;
  for (int e = 0; e < E; ++e) loads[e] = 0;
  for (int64_t p = 0; p < P; ++p) {
    int32_t e = topk[p];
    if (e < 0 || e >= E) {
      ++bad;
      continue;
    }
    loads[e] += 1;
  }
  int32_t mx = 0;
  for (int e = 0; e < E; ++e)
    if (loads[e] > mx) mx = loads[e];
  *max_vio = (P > 0) ? ((double)mx * (double)E) / (double)P - 1.0 : 0.0;
  return bad;
}

/* ------------------------------------------------------------- 2. plan */
/*
 * [GR] "Η βασική υπόσχεση του MoonEP: σταθερό φορτίο S × K" and [FR]
 * "Comment fonctionne MoonEP": every rank must end up processing exactly S*K
 * routed pairs, which the library reaches by planning a few temporary copies
 * (replicas) of hot experts on other ranks, online, from the current router
 * output.  [JA] "その仕組みは高速なエキスパート複製に依存する": the plan
 * decides which hot experts get copies, where each copy runs and how many
 * tokens each instance takes.  The pages do not print the rule; this library's
 * deterministic reading is:
 *   - home placement: expert e lives on rank floor(e / E_R) ([GR] "Το memory
 *     contract...": rows 0..E-1 hold the ranks' own experts);
 *   - rank load L_r = sum of T_e over its home experts; excess X_r = L_r - S*K
 *     when positive, deficit D_r = S*K - L_r when positive;
 *   - each overloaded rank (ascending r) cuts its excess into chunks taken from
 *     its home experts in DESCENDING id: chunk = min(T_e, remaining excess),
 *     empty chunks skipped, stop when the excess is used up;
 *   - the chunk sequence is matched against the deficit sequence (underloaded
 *     ranks in ascending r) by walking both in order: each step emits one
 *     replica (expert of the current chunk, rank of the current deficit,
 *     min(chunk left, deficit left)) and advances whichever is exhausted (both
 *     when they end together) -- the sequential form of a merge of the two
 *     prefix sums.  Emission order is the "match order".
 *   - home_count[e] = T_e minus the pairs its replicas take.
 *
 * Returns n_rep (>= 0), or -1 when sum(loads) != R*S*K.
 */
int oracle_plan(const int32_t* loads, int R, int64_t S, int K, int E, int32_t* rep_expert, int32_t* rep_rank,
                int32_t* rep_count, int32_t* home_count) {
  int ER = E / R;
  int64_t SK = S * (int64_t)K;
  int64_t total = 0;
  for (int e = 0; e < E; ++e) total += loads[e];
  if (total != (int64_t)R * SK) return -1;

  int64_t* L = (int64_t*)calloc((size_t)R, sizeof(int64_t));
  for (int e = 0; e < E; ++e) L[e / ER] += loads[e];

  /* supply: chunks (expert, size) */
  int32_t* ch_e = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int64_t* ch_n = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  int nch = 0;
  for (int r = 0; r < R; ++r) {
    int64_t rem = L[r] - SK;
    if (rem <= 0) continue;
    for (int e = (r + 1) * ER - 1; e >= r * ER && rem > 0; --e) {
      int64_t take = loads[e] < rem ? loads[e] : rem;
      if (take <= 0) continue;
      ch_e[nch] = e;
      ch_n[nch] = take;
      ++nch;
      rem -= take;
    }
  }
  /* demand: underloaded ranks (rank, deficit) */
  int32_t* dm_r = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
  int64_t* dm_n = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  int ndm = 0;
  for (int r = 0; r < R; ++r) {
    if (SK - L[r] > 0) {
      dm_r[ndm] = r;
      dm_n[ndm] = SK - L[r];
      ++ndm;
    }
  }
  /* two-pointer walk */
  int nrep = 0, i = 0, j = 0;
  int64_t left_c = nch ? ch_n[0] : 0, left_d = ndm ? dm_n[0] : 0;
  while (i < nch && j < ndm) {
    int64_t take = left_c < left_d ? left_c : left_d;
    rep_expert[nrep] = ch_e[i];
    rep_rank[nrep] = dm_r[j];
    rep_count[nrep] = (int32_t)take;
    ++nrep;
    left_c -= take;
    left_d -= take;
    if (left_c == 0) {
      ++i;
      if (i < nch) left_c = ch_n[i];
    }
    if (left_d == 0) {
      ++j;
      if (j < ndm) left_d = dm_n[j];
    }
  }
  for (int e = 0; e < E; ++e) home_count[e] = loads[e];
  for (int m = 0; m < nrep; ++m) home_count[rep_expert[m]] -= rep_count[m];

  free(L);
  free(ch_e);
  free(ch_n);
  free(dm_r);
  free(dm_n);
  return nrep;
}

/* ----------------------------------------------------------- 3. layout */
/*
 * [GR] "Online planning, zero copy και στατικά σχήματα": tokens are written
 * straight to their final positions, grouped by expert, in a static S*K buffer
 * per rank.  [JA] "UltraEPのMoE負荷分散はルーティング後に対応する": the
 * selected tokens are split between the original expert and its temporary
 * replicas.  Reading used here:
 *   - pairs of each expert are listed in ascending flattened index p (a stable
 *     grouping by expert, ties in (source rank, token, k) order);
 *   - the home copy takes the first home_count[e] pairs of e's list, then each
 *     replica of e, in match order, takes the next rep_count[m];
 *   - rank r's rows, from r*S*K on, hold its home experts in id order, then the
 *     replicas it receives in match order.
 * Global slot ids: e for the home copy of e, E + m for replica m.  slot_order
 * lists slot ids in buffer order; cu_seqlens[i] is the first row of the i-th
 * slot in that order, cu_seqlens[E + n_rep] = P.
 * pos[p] = row of pair p, src[row] = p, pair_slot[p] = slot id of pair p.
 * Pairs with an id outside [0, E) get pos = -1 and slot = -1.
 * Returns 0, or -1 if a rank's rows do not come out to S*K.
 */
int oracle_layout(const int32_t* topk, int64_t T, int K, int E, int R, int64_t S, int n_rep,
                  const int32_t* rep_expert, const int32_t* rep_rank, const int32_t* rep_count,
                  const int32_t* home_count, int32_t* pos, int32_t* src, int32_t* pair_slot, int32_t* slot_order,
                  int32_t* cu_seqlens) {
  int64_t P = T * (int64_t)K, SK = S * (int64_t)K;
  int ER = E / R;
  /* per-expert lists in ascending p */
  int64_t* start = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
  for (int64_t p = 0; p < P; ++p)
    if (topk[p] >= 0 && topk[p] < E) start[topk[p] + 1] += 1;
  for (int e = 0; e < E; ++e) start[e + 1] += start[e];
  int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  for (int e = 0; e < E; ++e) fill[e] = start[e];
  int32_t* list = (int32_t*)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
  for (int64_t p = 0; p < P; ++p) {
    pos[p] = -1;
    pair_slot[p] = -1;
    if (topk[p] >= 0 && topk[p] < E) list[fill[topk[p]]++] = (int32_t)p;
  }
  /* where each copy's range starts in its expert's list: the home copy at 0,
   * replica m after the home copy and the earlier replicas of the same expert */
  int64_t* next = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  for (int e = 0; e < E; ++e) next[e] = home_count[e];
  int64_t* rep_first = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_rep > 0 ? n_rep : 1));
  for (int m = 0; m < n_rep; ++m) {
    rep_first[m] = next[rep_expert[m]];
    next[rep_expert[m]] += rep_count[m];
  }
  int rc = 0, nslot = 0;
  for (int r = 0; r < R; ++r) {
    int64_t row = (int64_t)r * SK;
    for (int e = r * ER; e < (r + 1) * ER; ++e) {
      slot_order[nslot] = e;
      cu_seqlens[nslot] = (int32_t)row;
      ++nslot;
      for (int64_t i = 0; i < home_count[e]; ++i) {
        int32_t p = list[start[e] + i];
        pos[p] = (int32_t)row;
        src[row] = p;
        pair_slot[p] = e;
        ++row;
      }
    }
    for (int m = 0; m < n_rep; ++m) {
      if (rep_rank[m] != r) continue;
      int e = rep_expert[m];
      slot_order[nslot] = E + m;
      cu_seqlens[nslot] = (int32_t)row;
      ++nslot;
      for (int64_t i = 0; i < rep_count[m]; ++i) {
        int32_t p = list[start[e] + rep_first[m] + i];
        pos[p] = (int32_t)row;
        src[row] = p;
        pair_slot[p] = E + m;
        ++row;
      }
    }
    if (row != (int64_t)(r + 1) * SK) rc = -1;
  }
  cu_seqlens[nslot] = (int32_t)P;
  free(start);
  free(fill);
  free(list);
  free(next);
  free(rep_first);
  return rc;
}

/* ------------------------------------------------------- 4. align-sort */
/*
 * [ZH] MoE Align & Sort: sort the routed token ids by expert id and pad each
 * expert's group to a multiple of the block size, so the grouped GEMM can take
 * every block from a single expert; the result carries one expert id per block
 * and the padded total.  Readings: the ids sorted are flattened pair indices p
 * (consumers recover the token as p / K), stable in p; padding and the unused
 * tail hold the sentinel P; unused expert_ids entries hold -1; an expert with no
 * pairs gets no block.
 *   c_e = #pairs of e;  pc_e = ceil(c_e / block_m) * block_m;
 *   off_e = sum_{e' < e} pc_e';  num_tokens_post_pad = sum_e pc_e;
 *   sorted_ids[off_e + i] = i-th pair of e in ascending p, i < c_e.
 * Returns num_tokens_post_pad, or -1 if a capacity is too small.
 */
int64_t oracle_align_sort(const int32_t* topk, int64_t T, int K, int E, int block_m, int32_t* sorted_ids,
                          int64_t sorted_cap, int32_t* expert_ids, int64_t expert_ids_cap) {
  int64_t P = T * (int64_t)K;
  int64_t* cnt = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  for (int64_t p = 0; p < P; ++p)
    if (topk[p] >= 0 && topk[p] < E) cnt[topk[p]] += 1;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * ((size_t)E + 1));
  off[0] = 0;
  for (int e = 0; e < E; ++e) {
    int64_t padded = (cnt[e] + block_m - 1) / block_m * block_m;
    off[e + 1] = off[e] + padded;
  }
  int64_t total = off[E];
  if (total > sorted_cap || total / block_m > expert_ids_cap) {
    free(cnt);
    free(off);
    return -1;
  }
  for (int64_t i = 0; i < sorted_cap; ++i) sorted_ids[i] = (int32_t)P;
  for (int64_t b = 0; b < expert_ids_cap; ++b) expert_ids[b] = -1;
  int64_t* fill = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  for (int e = 0; e < E; ++e) fill[e] = off[e];
  for (int64_t p = 0; p < P; ++p)
    if (topk[p] >= 0 && topk[p] < E) sorted_ids[fill[topk[p]]++] = (int32_t)p;
  for (int e = 0; e < E; ++e)
    for (int64_t b = off[e] / block_m; b < off[e + 1] / block_m; ++b) expert_ids[b] = e;
  free(cnt);
  free(off);
  free(fill);
  return total;
}

/* --------------------------------------------------------- 5. dispatch */
/*
 * [GR] "Online planning, zero copy και στατικά σχήματα": each routed copy of a
 * token's hidden row is written straight into its final row of the expert-
 * grouped buffer.  buf[pos[p]] = x[p / K], bitwise, for every pair p with a
 * valid pos.
 */
void oracle_dispatch(const uint16_t* x, int64_t T, int K, int64_t H, const int32_t* pos, uint16_t* buf) {
  int64_t P = T * (int64_t)K;
  for (int64_t p = 0; p < P; ++p) {
    if (pos[p] < 0) continue;
    memcpy(buf + (int64_t)pos[p] * H, x + (p / K) * H, (size_t)H * 2);
  }
}

/* Stand-in for the expert computation (the grouped GEMM is outside the path):
 * y[row] = bf16_rn(float(buf[row]) * s[e]) with e the logical expert of the row,
 * found through src: e = topk[src[row]]. */
void oracle_expert_standin(const uint16_t* buf, int64_t nrows, int64_t H, const int32_t* src, const int32_t* topk,
                           const float* scale, uint16_t* y) {
  for (int64_t row = 0; row < nrows; ++row) {
    float s = scale[topk[src[row]]];
    for (int64_t h = 0; h < H; ++h) {
      float v = bf16_to_f32(buf[row * H + h]) * s;
      y[row * H + h] = f32_to_bf16(v);
    }
  }
}

/* ---------------------------------------------------------- 6. combine */
/*
 * [GR] "Τι δείχνουν — και τι δεν αποδεικνύουν — τα benchmarks" names combine
 * among the steps of the layer: the K expert outputs of each token are brought
 * back and weighted by the gate.  out[t] = bf16_rn( sum_{k=0..K-1} w[t,k] *
 * float(y[pos[t*K+k]]) ), accumulated in fp32 in k order from 0.0f, each
 * product and each sum rounded separately, one final rounding to bf16.
 * Pairs with pos < 0 contribute nothing.
 */
void oracle_combine(const uint16_t* y, const float* w, const int32_t* pos, int64_t T, int K, int64_t H,
                    uint16_t* out) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int k = 0; k < K; ++k) {
        int32_t row = pos[t * K + k];
        if (row < 0) continue;
        float prod = w[t * K + k] * bf16_to_f32(y[(int64_t)row * H + h]);
        acc = acc + prod;
      }
      out[t * H + h] = f32_to_bf16(acc);
    }
  }
}

/*
 * Combine for the stand-in expert in closed form.  Because the stand-in's
 * output row depends only on the token and the logical expert, combine's
 * result does not depend on the plan or the layout:
 *   out[t] = bf16_rn( sum_k w[t,k] * float(bf16_rn(float(x[t]) * s[e_k])) ).
 * Rows of x, w and topk are given for nt selected tokens (row i = token i of
 * the selection), so the check streams at any workload size.
 */
void oracle_combine_closed(const uint16_t* x_rows, const float* w_rows, const int32_t* topk_rows, int64_t nt,
                           int K, int64_t H, const float* scale, uint16_t* out) {
  for (int64_t i = 0; i < nt; ++i) {
    for (int64_t h = 0; h < H; ++h) {
      float xv = bf16_to_f32(x_rows[i * H + h]);
      float acc = 0.0f;
      for (int k = 0; k < K; ++k) {
        float yv = bf16_to_f32(f32_to_bf16(xv * scale[topk_rows[i * K + k]]));
        float prod = w_rows[i * K + k] * yv;
        acc = acc + prod;
      }
      out[i * H + h] = f32_to_bf16(acc);
    }
  }
}

/* ------------------------------------------------------ 7. grad reduce */
/*
 * [GR] "Τι συμβαίνει στους gradients κατά την εκπαίδευση": gradients are kept
 * in fp32; replica slots write to a separate reduce buffer, and reduce_grad
 * adds the slots belonging to a rank's own experts into the local parameter
 * gradient and then clears the used slots.  [JA]: replica gradients are folded
 * back into the primary expert.  Order used: for every element, the home value
 * first, then each replica of that expert in match order, one fp32 add each:
 *   g_home[e][j] = ((g_home[e][j] + g_rep[m1][j]) + g_rep[m2][j]) + ...
 * rep_dtype 0: g_rep is fp32; 1: bf16 (widened exactly to fp32 before the add).
 * clear != 0 zeroes each used replica row afterwards.
 */
void oracle_grad_reduce(float* g_home, void* g_rep, int rep_dtype, int64_t n, int n_rep, const int32_t* rep_expert,
                        int clear) {
  for (int m = 0; m < n_rep; ++m) {
    float* dst = g_home + (int64_t)rep_expert[m] * n;
    if (rep_dtype == 0) {
      float* g = (float*)g_rep + (int64_t)m * n;
      for (int64_t j = 0; j < n; ++j) dst[j] = dst[j] + g[j];
      if (clear) memset(g, 0, (size_t)n * 4);
    } else {
      uint16_t* g = (uint16_t*)g_rep + (int64_t)m * n;
      for (int64_t j = 0; j < n; ++j) dst[j] = dst[j] + bf16_to_f32(g[j]);
      if (clear) memset(g, 0, (size_t)n * 2);
    }
  }
}

/* ------------------------------------------------------ 8. backward */
/*
 * The MoE Align & Sort report [ZH] recalls that the permute which records the
 * source -> destination mapping has unpermute as its gradient.  Dispatch is
 * that permute (every token row copied to K rows) and combine its weighted
 * inverse, so their gradients are:
 *
 * backward of dispatch (unpermute): dx[t] = bf16_rn( sum_{k=0..K-1}
 *   float(dbuf[pos[t*K+k]]) ), accumulated in fp32 in k order from 0, one add
 *   per term, one rounding to bf16.  Pairs with pos < 0 contribute nothing.
 */
void oracle_dispatch_backward(const uint16_t* dbuf, const int32_t* pos, int64_t T, int K, int64_t H, uint16_t* dx) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) {
      float acc = 0.0f;
      for (int k = 0; k < K; ++k) {
        int32_t row = pos[t * K + k];
        if (row < 0) continue;
        acc = acc + bf16_to_f32(dbuf[(int64_t)row * H + h]);
      }
      dx[t * H + h] = f32_to_bf16(acc);
    }
  }
}

/*
 * backward of combine, given dout [T, H] (bf16):
 *   dy[pos[t*K+k]] = bf16_rn( w[t,k] * float(dout[t]) )   one fp32 multiply per element;
 *   dw[t,k] = sum_h float(dout[t,h]) * float(y[pos[t*K+k], h])
 * dw is accumulated in fp64 (each product of two bf16 values is exact in fp64;
 * the sum carries only fp64 rounding), the reference against which an fp32
 * reduction in any order is bounded.  Rows of dy not addressed by any pair are
 * left untouched.
 */
void oracle_combine_backward(const uint16_t* dout, const float* w, const uint16_t* y, const int32_t* pos, int64_t T,
                             int K, int64_t H, uint16_t* dy, double* dw) {
  for (int64_t t = 0; t < T; ++t) {
    for (int k = 0; k < K; ++k) {
      int32_t row = pos[t * K + k];
      if (row < 0) {
        dw[t * K + k] = 0.0;
        continue;
      }
      double s = 0.0;
      for (int64_t h = 0; h < H; ++h) {
        float g = bf16_to_f32(dout[t * H + h]);
        dy[(int64_t)row * H + h] = f32_to_bf16(w[t * K + k] * g);
        s += (double)g * (double)bf16_to_f32(y[(int64_t)row * H + h]);
      }
      dw[t * K + k] = s;
    }
  }
}

/* ------------------------------------------------ 9. prefetch slots */
/*
 * [GR] "Το memory contract που πρέπει να καταλάβει η τεχνική ομάδα": each rank's
 * grouped-GEMM weight tensor is [E+B, H, H'], rows 0..E-1 for the ranks' own
 * experts and rows E..E+B-1 as local prefetch slots; when a rank needs more
 * remote experts than it has slots, the rest are read from their home rank
 * (correct, slower).  Reading used: replicas take a rank's slots in match order,
 * so the j-th replica a rank receives gets slot E + j while j < B, and -1
 * (read from the home rank) after that.  The token layout does not change.
 * slot[m] for m < n_rep; n_remote[r] = replicas rank r reads from home.
 *
 * load_capped (may be NULL): the other reading of the overflow, where a
 * replica without a slot is not made at all and its pairs stay with the
 * expert's home rank e / (E/R).  Rank r then holds S*K, less the pairs of its
 * own slotless replicas, plus the pairs of slotless replicas of its experts.
 * B = 0 gives back the unplanned rank loads; B >= every rank's replica count
 * gives S*K everywhere.
 */
void oracle_prefetch_slots(int n_rep, const int32_t* rep_expert, const int32_t* rep_rank, const int32_t* rep_count,
                           int E, int R, int64_t SK, int B, int32_t* slot, int32_t* n_remote, int64_t* load_capped) {
  int32_t* seen = (int32_t*)calloc((size_t)R, sizeof(int32_t));
  int ER = E / R;
  for (int r = 0; r < R; ++r) {
    n_remote[r] = 0;
    if (load_capped) load_capped[r] = SK;
  }
  for (int m = 0; m < n_rep; ++m) {
    int r = rep_rank[m];
    int j = seen[r]++;
    if (j < B) {
      slot[m] = E + j;
    } else {
      slot[m] = -1;
      n_remote[r] += 1;
      if (load_capped) {
        load_capped[r] -= rep_count[m];
        load_capped[rep_expert[m] / ER] += rep_count[m];
      }
    }
  }
  free(seen);
}

/* ----------------------------------------------- 10. quota planner */
/*
 * [JA] "その仕組みは高速なエキスパート複製に依存する" (remio.ai UltraEP article):
 * planning starts from the exact load matrix produced by routing (how many
 * tokens of each source rank chose each logical expert); a target load
 * threshold is searched for that keeps every rank below it within the replica
 * slots available; a quota-driven planner then decides in one step which heavy
 * experts get copies, on which ranks, and how many tokens each instance takes;
 * a copy exists only when it is given work; tokens use the capacity of a local
 * instance before the rest of the demand is sent elsewhere; the aggregated
 * quotas become per-token destinations by a lookup on cumulative quotas.
 *
 * The page prints no formula.  Readings used here:
 *   - source rank of pair p = p / (S*K); home rank of expert e = e / E_R;
 *     H_r = sum of T_e over rank r's home experts;
 *   - at threshold tau, rank r sheds X_r = max(0, H_r - tau) pairs, taken from
 *     its home experts HEAVIEST FIRST (ties: lower id), chunk = min(T_e, excess
 *     left); rank r has room C_r = max(0, tau - H_r);
 *   - chunks (overloaded ranks ascending) are matched to rooms (ranks
 *     ascending) as in the MoonEP walk, one replica per match, except that a
 *     rank stops taking pieces once it holds B of them (its slot budget);
 *     tau is feasible when every chunk is placed;
 *   - tau* is the smallest feasible tau from ceil(P/R) up (the largest H_r is
 *     always feasible: nothing is shed);
 *   - instances of expert e: its home copy, then its replicas in match order;
 *     instance i on rank r_i with quota q_i first takes its local pairs -- the
 *     first min(q_i, L[r_i][e]) pairs of e from source rank r_i, in pair order
 *     -- and the remaining pairs of e, in pair order, fill the instances' left
 *     quotas by cumulative lookup in instance order;
 *   - layout: rank r's rows follow rank r-1's (each rank holds its load, at
 *     most tau*); within a rank, home experts in id order then received
 *     replicas in match order; within an instance, local pairs then looked-up
 *     pairs, each in pair order.
 */

/* Lm[s*E + e] = pairs of source rank s (pairs [s*SK, (s+1)*SK)) routed to e. */
void oracle_load_matrix(const int32_t* topk, int R, int64_t SK, int E, int32_t* Lm) {
  for (int64_t i = 0; i < (int64_t)R * E; ++i) Lm[i] = 0;
  for (int64_t p = 0; p < (int64_t)R * SK; ++p) {
    int e = topk[p];
    if (e >= 0 && e < E) Lm[(p / SK) * E + e] += 1;
  }
}

/*
 * The quota plan at threshold tau with at most B replicas per rank.  Returns
 * n_rep, or -1 when tau is not feasible.  rep_* hold at least E + R - 1 entries.
 */
int oracle_quota_plan_at(const int32_t* loads, int E, int R, int64_t tau, int B, int32_t* rep_expert,
                         int32_t* rep_rank, int32_t* rep_count, int32_t* home_quota) {
  int ER = E / R;
  int64_t* H = (int64_t*)calloc((size_t)R, sizeof(int64_t));
  for (int e = 0; e < E; ++e) H[e / ER] += loads[e];

  /* chunks: overloaded ranks ascending, each rank's experts heaviest first */
  int32_t* ch_e = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int64_t* ch_n = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
  char* used = (char*)calloc((size_t)E, 1);
  int nch = 0;
  for (int r = 0; r < R; ++r) {
    int64_t rem = H[r] - tau;
    while (rem > 0) {
      int best = -1;
      for (int e = r * ER; e < (r + 1) * ER; ++e)
        if (!used[e] && (best < 0 || loads[e] > loads[best])) best = e;
      if (best < 0 || loads[best] <= 0) break;
      used[best] = 1;
      int64_t take = loads[best] < rem ? loads[best] : rem;
      ch_e[nch] = best;
      ch_n[nch] = take;
      ++nch;
      rem -= take;
    }
  }
  /* rooms: ranks below tau, ascending */
  int32_t* rm_r = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
  int64_t* rm_n = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
  int nrm = 0;
  for (int r = 0; r < R; ++r) {
    if (tau - H[r] > 0) {
      rm_r[nrm] = r;
      rm_n[nrm] = tau - H[r];
      ++nrm;
    }
  }
  /* the walk; a room closes when full or when it holds B pieces */
  int nrep = 0, i = 0, j = 0, pieces = 0;
  int64_t left_c = nch ? ch_n[0] : 0, left_r = nrm ? rm_n[0] : 0;
  if (B <= 0) j = nrm; /* no slot anywhere */
  while (i < nch && j < nrm) {
    int64_t take = left_c < left_r ? left_c : left_r;
    rep_expert[nrep] = ch_e[i];
    rep_rank[nrep] = rm_r[j];
    rep_count[nrep] = (int32_t)take;
    ++nrep;
    ++pieces;
    left_c -= take;
    left_r -= take;
    if (left_c == 0) {
      ++i;
      if (i < nch) left_c = ch_n[i];
    }
    if (left_r == 0 || pieces == B) {
      ++j;
      pieces = 0;
      if (j < nrm) left_r = rm_n[j];
    }
  }
  int ok = (i == nch);
  if (ok) {
    for (int e = 0; e < E; ++e) home_quota[e] = loads[e];
    for (int m = 0; m < nrep; ++m) home_quota[rep_expert[m]] -= rep_count[m];
  }
  free(H);
  free(ch_e);
  free(ch_n);
  free(used);
  free(rm_r);
  free(rm_n);
  return ok ? nrep : -1;
}

/* tau*: the smallest feasible threshold from ceil(P/R) up. */
int64_t oracle_quota_threshold(const int32_t* loads, int E, int R, int64_t P, int B) {
  int cap = E + R - 1;
  int32_t* a = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* b = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* c = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
  int32_t* h = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
  int64_t tau = (P + R - 1) / R;
  while (oracle_quota_plan_at(loads, E, R, tau, B, a, b, c, h) < 0) ++tau;
  free(a);
  free(b);
  free(c);
  free(h);
  return tau;
}

/*
 * Per-pair destinations of a quota plan.  pos[p] = row of pair p, src[row] = p,
 * slot_order / cu_seqlens over the E + n_rep slots in buffer order (slot id e
 * for e's home copy, E + m for replica m), rank_load[r] = rows of rank r,
 * *n_local = pairs placed on their own source rank.  Returns 0, -1 when an
 * expert would have two instances on one rank or a quota goes negative, -2 on
 * an expert id outside [0, E).
 */
int oracle_quota_layout(const int32_t* topk, int R, int64_t SK, int E, int n_rep, const int32_t* rep_expert,
                        const int32_t* rep_rank, const int32_t* rep_count, const int32_t* home_quota, int32_t* pos,
                        int32_t* src, int32_t* slot_order, int32_t* cu_seqlens, int32_t* rank_load,
                        int64_t* n_local) {
  int ER = E / R;
  int64_t P = (int64_t)R * SK;
  int n_inst = E + n_rep;
  for (int64_t p = 0; p < P; ++p)
    if (topk[p] < 0 || topk[p] >= E) return -2;
  int32_t* Lm = (int32_t*)malloc(sizeof(int32_t) * (size_t)R * (size_t)E);
  oracle_load_matrix(topk, R, SK, E, Lm);

  int32_t* ie = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_inst); /* expert */
  int32_t* ir = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_inst); /* rank */
  int64_t* iq = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_inst); /* quota */
  int64_t* il = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_inst); /* local pairs */
  int64_t* ic = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_inst); /* cumulative left quota before it */
  int64_t* ib = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_inst); /* first row */
  int32_t* at = (int32_t*)malloc(sizeof(int32_t) * (size_t)E * (size_t)R); /* instance of e on r */
  int32_t* lst = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_inst);        /* instances grouped by expert */
  int32_t* lst_off = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
  int64_t* seen_se = (int64_t*)calloc((size_t)R * (size_t)E, sizeof(int64_t));
  int64_t* seen_e = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  int64_t* rl = (int64_t*)calloc((size_t)R, sizeof(int64_t));
  int rc = 0;

  for (int e = 0; e < E; ++e) {
    ie[e] = e;
    ir[e] = e / ER;
    iq[e] = home_quota[e];
  }
  for (int m = 0; m < n_rep; ++m) {
    ie[E + m] = rep_expert[m];
    ir[E + m] = rep_rank[m];
    iq[E + m] = rep_count[m];
  }
  for (int64_t k = 0; k < (int64_t)E * R; ++k) at[k] = -1;
  for (int i = 0; i < n_inst; ++i) {
    if (iq[i] < 0 || at[ie[i] * R + ir[i]] >= 0) rc = -1;
    at[ie[i] * R + ir[i]] = i;
    il[i] = iq[i] < Lm[ir[i] * E + ie[i]] ? iq[i] : Lm[ir[i] * E + ie[i]];
    lst_off[ie[i] + 1] += 1;
  }
  if (rc == 0) {
    /* instance lists per expert: home first, then replicas in match order */
    for (int e = 0; e < E; ++e) lst_off[e + 1] += lst_off[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int i = 0; i < n_inst; ++i) lst[lst_off[ie[i]] + fill[ie[i]]++] = i;
    free(fill);
    for (int e = 0; e < E; ++e) {
      int64_t run = 0;
      for (int k = lst_off[e]; k < lst_off[e + 1]; ++k) {
        ic[lst[k]] = run;
        run += iq[lst[k]] - il[lst[k]];
      }
    }
    /* rows: ranks in order; home experts by id, then received replicas by m */
    for (int i = 0; i < n_inst; ++i) rl[ir[i]] += iq[i];
    int64_t row = 0;
    int ns = 0;
    cu_seqlens[0] = 0;
    for (int r = 0; r < R; ++r) {
      for (int e = r * ER; e < (r + 1) * ER; ++e) {
        ib[e] = row;
        row += iq[e];
        slot_order[ns] = e;
        cu_seqlens[++ns] = (int32_t)row;
      }
      for (int m = 0; m < n_rep; ++m) {
        if (rep_rank[m] != r) continue;
        ib[E + m] = row;
        row += iq[E + m];
        slot_order[ns] = E + m;
        cu_seqlens[++ns] = (int32_t)row;
      }
      rank_load[r] = (int32_t)rl[r];
    }
    /* pairs in order: local first, then the cumulative-quota lookup */
    *n_local = 0;
    for (int64_t p = 0; p < P; ++p) {
      int e = topk[p];
      int s = (int)(p / SK);
      int64_t ls = seen_se[(int64_t)s * E + e]++;
      int i = at[e * R + s];
      int64_t r;
      if (i >= 0 && ls < il[i]) {
        r = ib[i] + ls;
        *n_local += 1;
      } else {
        int64_t jj = seen_e[e]++;
        r = -1;
        for (int k = lst_off[e]; k < lst_off[e + 1]; ++k) {
          int c = lst[k];
          if (jj >= ic[c] && jj < ic[c] + (iq[c] - il[c])) {
            r = ib[c] + il[c] + (jj - ic[c]);
            break;
          }
        }
        if (r < 0) {
          rc = -1;
          break;
        }
      }
      pos[p] = (int32_t)r;
      src[r] = (int32_t)p;
    }
  }
  free(Lm);
  free(ie);
  free(ir);
  free(iq);
  free(il);
  free(ic);
  free(ib);
  free(at);
  free(lst);
  free(lst_off);
  free(seen_se);
  free(seen_e);
  free(rl);
  return rc;
}
