/*
 * CPU oracle for the MoE routing path.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, single-threaded C with one loop per definition.  Only the test
 * suite, the package's smoke check and the benchmark's CPU-baseline leg may
 * load or run this; the CUDA library never does, and this file shares no code,
 * header, table or helper with it.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off (no fast-math) -shared -fPIC -lm.
 * fp32 steps use IEEE single precision with libm expf and IEEE '/'; where a
 * result has a plain real-valued definition (sums, dot products, RMS) it is
 * accumulated in double and rounded once.
 *
 * Pages cited (by title and section):
 *   [TE]   Implementation:NVIDIA TransformerEngine Fused Router
 *   [TRT]  flashinfer.fused_moe.trtllm_gen_routing
 *   [NKI]  RMSNorm Router Top-K A2AV Kernel API Reference
 *   [LMD]  Implementation:InternLM Lmdeploy Gemm MoeUtils
 *   [MAX]  max.nn.moe.SigmoidTopKRouter
 *
 * Readings where the pages are silent are marked READING and listed in the
 * design notes.  "parity unpinned": the sigmoid branch of the aux scores
 * (normalised sigmoid) is pinned only by closed forms (uniform rows, and rows
 * whose sigmoids are exact: 0, 1/2, 1).
 *
 * Return codes: 0 ok, -1 invalid argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_SOFTMAX 0
#define ORC_SIGMOID 1

/* ---- bf16 <-> fp32 (IEEE 754 binary32 truncated to its top 16 bits) ---- */

/* bf16 -> fp32 is exact: the 16 bits are the high half of the binary32 pattern. */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on the 16 dropped bits
 * (IEEE 754 roundTiesToEven).  NaN stays NaN (quiet bit set). */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
    return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* double -> bf16 with a single rounding (nearest, ties to even): round to odd
 * at fp32 precision, then to nearest-even at bf16 precision.  Rounding to odd
 * at >= 2 extra bits followed by round-to-nearest equals direct
 * round-to-nearest (Boldo & Melquiond, "Emulation of FMA and correctly rounded
 * sums: proved algorithms using rounding to odd", IEEE TC 2008). */
static uint16_t f64_to_bf16(double y) {
  float f = (float)y;
  if ((double)f != y && isfinite(f)) {
    if (fabs((double)f) > fabs(y)) f = nextafterf(f, 0.0f);
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u |= 1u;
    memcpy(&f, &u, sizeof f);
  }
  return f32_to_bf16(f);
}

float oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }
uint16_t oracle_f64_to_bf16(double y) { return f64_to_bf16(y); }
uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16(f); }

static float load_elem(const void* p, int dtype, size_t i) {
  if (dtype == ORC_BF16) return bf16_to_f32(((const uint16_t*)p)[i]);
  return ((const float*)p)[i];
}

/* ---- score functions [TE: I/O Contract, score_function; MAX: step 2] ---- */

/* sigmoid in fp32: 1 / (1 + exp(-x)). */
static float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

/* softmax over n values in fp32: max, exp of the shifted values, sum in index
 * order, divide. */
static void softmax_f32(const float* x, int n, float* out) {
  float m = x[0];
  for (int i = 1; i < n; ++i)
    if (x[i] > m) m = x[i];
  float s = 0.0f;
  for (int i = 0; i < n; ++i) {
    out[i] = expf(x[i] - m);
    s = s + out[i];
  }
  for (int i = 0; i < n; ++i) out[i] = out[i] / s;
}

/* "a beats b": larger key first, equal keys -> lower index first. */
static int beats(float ka, int a, float kb, int b) {
  if (ka > kb) return 1;
  if (ka < kb) return 0;
  return a < b;
}

/* Pick the k best entries of keys[0..n) among those with allowed[i] != 0,
 * best first, by (key desc, index asc).  Returns the number picked. */
static int pick_topk(const float* keys, const unsigned char* allowed, int n, int k, int* out) {
  unsigned char* taken = (unsigned char*)calloc((size_t)n, 1);
  int got = 0;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int i = 0; i < n; ++i) {
      if (taken[i] || (allowed && !allowed[i])) continue;
      if (best < 0 || beats(keys[i], i, keys[best], best)) best = i;
    }
    if (best < 0) break;
    taken[best] = 1;
    out[got++] = best;
  }
  free(taken);
  return got;
}

static int is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

static int groups_enabled(int n_group, int topk_group) { return n_group > 1 && topk_group > 0; }

/*
 * Expert selection and routing weights for T tokens.
 *
 * score_fn / softmax_before_topk  [TE: I/O Contract, score_function and
 *   use_pre_softmax; NKI: Notes, ACT2 pipeline]:
 *     softmax, pre : s = softmax(logits), key = s + b
 *     sigmoid      : s = sigmoid(logit),  key = s + b        [MAX: steps 2-3]
 *     post (either): key = logit + b; the score function is applied to the k
 *                    selected logits only (softmax over the k, or sigmoid each)
 *   b is the expert / correction bias (0 without one); it enters the key only
 *   [MAX: steps 3-4; TRT: routing_bias].
 * Groups [TRT: n_group, topk_group; TE: num_groups, group_topk]: with
 *   n_group > 1 and topk_group > 0 the E experts form n_group contiguous groups;
 *   a group's score is the sum of its group_score_topn largest keys (largest
 *   first, fp32 adds); groups are ranked by (score desc, group asc) and the
 *   first topk_group kept; experts outside kept groups cannot be selected.
 *   READING: the group score rule (sum of top-n keys) is the DeepSeek-V3 rule
 *   the grouped workload states; the pages name the parameters only.
 * Top-k: the k best allowed experts by (key desc, expert asc); that order is
 *   the slot order.
 * Weights [MAX: step 4; TRT: norm_topk_prob, routed_scaling_factor]:
 *   v_j = unbiased score of the selected expert (post: the score function over
 *   the selected logits); with renormalize, w_j = v_j / sum_j v_j * scale
 *   (sum in slot order), otherwise w_j = v_j * scale.
 *
 * Outputs: ids [T,k] int32, weights [T,k] fp32 (callers round to bf16 where
 * the weights are stored in bf16), keys [T,E] (optional), group scores
 * [T,n_group] (optional), kept-group flags [T,n_group] (optional).
 */
int oracle_route_select(int T, int E, int k, int score_fn, int softmax_before_topk,
                        int n_group, int topk_group, int group_topn, int renormalize,
                        float scale, const void* logits, int logits_dtype, const void* bias,
                        int bias_dtype, int32_t* ids, float* weights, float* keys_out,
                        float* gscore_out, unsigned char* gkept_out) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  int grouped = groups_enabled(n_group, topk_group);
  int gs = 0;
  if (grouped) {
    if (E % n_group != 0 || group_topn <= 0) return -1;
    gs = E / n_group;
    if (group_topn > gs) return -1;
    int kept = topk_group < n_group ? topk_group : n_group;
    if (k > kept * gs) return -1;
  }
  float* l = (float*)malloc(sizeof(float) * (size_t)E);
  float* s = (float*)malloc(sizeof(float) * (size_t)E);
  float* key = (float*)malloc(sizeof(float) * (size_t)E);
  unsigned char* allowed = (unsigned char*)malloc((size_t)E);
  int* sel = (int*)malloc(sizeof(int) * (size_t)k);
  float* v = (float*)malloc(sizeof(float) * (size_t)k);
  float* gsc = (float*)malloc(sizeof(float) * (size_t)(n_group > 0 ? n_group : 1));
  int* gsel = (int*)malloc(sizeof(int) * (size_t)(n_group > 0 ? n_group : 1));
  int* tmp = (int*)malloc(sizeof(int) * (size_t)E);
  int post = !softmax_before_topk;

  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) l[e] = load_elem(logits, logits_dtype, (size_t)t * E + e);
    if (post) {
      for (int e = 0; e < E; ++e) s[e] = l[e];
    } else if (score_fn == ORC_SOFTMAX) {
      softmax_f32(l, E, s);
    } else {
      for (int e = 0; e < E; ++e) s[e] = sigmoid_f32(l[e]);
    }
    for (int e = 0; e < E; ++e) {
      float b = bias ? load_elem(bias, bias_dtype, (size_t)e) : 0.0f;
      key[e] = s[e] + b;
      allowed[e] = 1;
    }
    if (keys_out) memcpy(keys_out + (size_t)t * E, key, sizeof(float) * (size_t)E);

    if (grouped) {
      for (int g = 0; g < n_group; ++g) {
        int got = pick_topk(key + (size_t)g * gs, NULL, gs, group_topn, tmp);
        float acc = key[g * gs + tmp[0]];
        for (int i = 1; i < got; ++i) acc = acc + key[g * gs + tmp[i]];
        gsc[g] = acc;
      }
      int kept = topk_group < n_group ? topk_group : n_group;
      pick_topk(gsc, NULL, n_group, kept, gsel);
      memset(allowed, 0, (size_t)E);
      for (int i = 0; i < kept; ++i)
        for (int e = gsel[i] * gs; e < (gsel[i] + 1) * gs; ++e) allowed[e] = 1;
      if (gscore_out) memcpy(gscore_out + (size_t)t * n_group, gsc, sizeof(float) * (size_t)n_group);
      if (gkept_out) {
        memset(gkept_out + (size_t)t * n_group, 0, (size_t)n_group);
        for (int i = 0; i < kept; ++i) gkept_out[(size_t)t * n_group + gsel[i]] = 1;
      }
    }
    pick_topk(key, allowed, E, k, sel);

    if (post) {
      float* sl = (float*)malloc(sizeof(float) * (size_t)k);
      for (int j = 0; j < k; ++j) sl[j] = l[sel[j]];
      if (score_fn == ORC_SOFTMAX) {
        softmax_f32(sl, k, v);
      } else {
        for (int j = 0; j < k; ++j) v[j] = sigmoid_f32(sl[j]);
      }
      free(sl);
    } else {
      for (int j = 0; j < k; ++j) v[j] = s[sel[j]];
    }
    if (renormalize) {
      float sum = 0.0f;
      for (int j = 0; j < k; ++j) sum = sum + v[j];
      for (int j = 0; j < k; ++j) v[j] = (v[j] / sum) * scale;
    } else {
      for (int j = 0; j < k; ++j) v[j] = v[j] * scale;
    }
    for (int j = 0; j < k; ++j) {
      ids[(size_t)t * k + j] = sel[j];
      weights[(size_t)t * k + j] = v[j];
    }
  }
  free(l); free(s); free(key); free(allowed); free(sel); free(v); free(gsc); free(gsel); free(tmp);
  return 0;
}

/* Upper bounds of the padded row count and of the tile count, used to size the
 * permutation outputs: every expert with at least one row pads by < tile. */
int oracle_route_capacity(int T, int E, int k, int tile, int64_t* max_padded, int64_t* max_tiles) {
  if (T < 0 || E <= 0 || k <= 0 || !is_pow2(tile)) return -1;
  int64_t rows = (int64_t)T * k;
  int64_t nz = rows < E ? rows : E;
  *max_padded = rows + nz * (tile - 1);
  *max_tiles = *max_padded / tile;
  return 0;
}

/*
 * Permutation bookkeeping for a grouped GEMM [TRT: Returns; Notes; LMD:
 * invokeMoeGate_V2 offsets and maps], for the experts of one expert-parallel
 * shard [TRT: Parameters, local_expert_offset / local_num_experts; Notes: a
 * tile's expert is its batch index + local_expert_offset].  Expert e is local
 * when off <= e < off + nl; its local index is le = e - off (off = 0, nl = E:
 * every expert, the single-GPU case).
 *   counts[le]     = number of (t, j) with ids[t,j] == off + le
 *   padded_le      = ceil(counts[le] / tile) * tile        (tile a power of two)
 *   offsets[0] = 0, offsets[le+1] = offsets[le] + padded_le;  P = offsets[nl]
 *   e2p[t*k + j]   = offsets[le] + (number of earlier (t', j') in token-major
 *                    order routed to the same expert)  -- slots follow token
 *                    order; -1 when ids[t,j] is not local (READING)
 *   p2t[p]         = t for every filled slot, -1 on padding (READING)
 *   for tile c in [0, P / tile): tile_expert[c] = the le whose padded range
 *                    holds row c*tile (the batch index); tile_mn_limit[c] =
 *                    min((c+1)*tile, offsets[le] + counts[le])  (READING:
 *                    exclusive end row)
 *   totals = {P, P / tile}
 * Entries of p2t at or past P and of the tile tables at or past P/tile are
 * left as the caller filled them.
 */
/*
 * With S fused shared experts [TRT: Parameters num_fused_shared_experts --
 * extra shared-expert slots appended per token, DeepSeekV3 path].  READING:
 * shared expert s has id E + s; it is local on every expert-parallel shard and
 * is indexed after the shard's routed experts (local index nl + s), so the
 * bookkeeping runs over nl + S local experts.  ids [T, k] may hold E .. E+S-1.
 */
int oracle_route_bookkeeping_shared(int T, int E, int S, int k, int tile, int off, int nl, const int32_t* ids,
                                    int32_t* counts, int32_t* offsets, int32_t* e2p, int32_t* p2t,
                                    int32_t* tile_expert, int32_t* tile_mn_limit, int32_t* totals) {
  if (T < 0 || E <= 0 || S < 0 || k <= 0 || !is_pow2(tile)) return -1;
  if (off < 0 || nl <= 0 || off + nl > E) return -1;
  const int NL = nl + S;  /* local experts: the shard's routed ones, then the shared ones */
  for (int le = 0; le < NL; ++le) counts[le] = 0;
  for (int64_t i = 0; i < (int64_t)T * k; ++i) {
    int e = ids[i];
    if (e < 0 || e >= E + S) return -1;
    if (e >= E) counts[nl + (e - E)] += 1;
    else if (e >= off && e < off + nl) counts[e - off] += 1;
  }
  offsets[0] = 0;
  for (int le = 0; le < NL; ++le) {
    int32_t padded = ((counts[le] + tile - 1) / tile) * tile;
    offsets[le + 1] = offsets[le] + padded;
  }
  int32_t P = offsets[NL];
  for (int32_t p = 0; p < P; ++p) p2t[p] = -1;
  int32_t* running = (int32_t*)calloc((size_t)NL, sizeof(int32_t));
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      int e = ids[(size_t)t * k + j];
      int le;
      if (e >= E) {
        le = nl + (e - E);
      } else if (e >= off && e < off + nl) {
        le = e - off;
      } else {
        e2p[(size_t)t * k + j] = -1;
        continue;
      }
      int32_t slot = offsets[le] + running[le];
      running[le] += 1;
      e2p[(size_t)t * k + j] = slot;
      p2t[slot] = t;
    }
  }
  free(running);
  int32_t ntiles = P / tile;
  for (int32_t c = 0; c < ntiles; ++c) {
    int32_t row = c * tile;
    int le = 0;
    while (!(offsets[le] <= row && row < offsets[le + 1])) ++le;  /* le < NL */
    int32_t lim = (c + 1) * tile;
    int32_t valid_end = offsets[le] + counts[le];
    tile_expert[c] = le;
    tile_mn_limit[c] = lim < valid_end ? lim : valid_end;
  }
  totals[0] = P;
  totals[1] = ntiles;
  return 0;
}

int oracle_route_bookkeeping(int T, int E, int k, int tile, int off, int nl, const int32_t* ids,
                             int32_t* counts, int32_t* offsets, int32_t* e2p, int32_t* p2t,
                             int32_t* tile_expert, int32_t* tile_mn_limit, int32_t* totals) {
  return oracle_route_bookkeeping_shared(T, E, 0, k, tile, off, nl, ids, counts, offsets, e2p, p2t, tile_expert,
                                         tile_mn_limit, totals);
}

/*
 * The fused shared-expert slots [TRT: Parameters num_fused_shared_experts].
 * READING: each token's S extra slots follow its k routed slots in order;
 * slot k + s holds expert E + s with weight 1.0 (the shared experts take no
 * part in selection, renormalisation or the routed scaling factor).
 */
int oracle_append_shared(int T, int k, int S, int E, const int32_t* ids, const float* weights, int32_t* ids_out,
                         float* weights_out) {
  if (T < 0 || k <= 0 || S < 0 || E <= 0) return -1;
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      ids_out[(size_t)t * (k + S) + j] = ids[(size_t)t * k + j];
      weights_out[(size_t)t * (k + S) + j] = weights[(size_t)t * k + j];
    }
    for (int s = 0; s < S; ++s) {
      ids_out[(size_t)t * (k + S) + k + s] = E + s;
      weights_out[(size_t)t * (k + S) + k + s] = 1.0f;
    }
  }
  return 0;
}

/*
 * Scores and routing map for the load-balancing loss [TE: Description,
 * fused_compute_score_for_moe_aux_loss; Signature].
 *   probs = softmax(logits) over E (fp32, as above); READING for sigmoid:
 *           s = sigmoid(logit), probs = s / sum_e s (parity unpinned beyond
 *           closed forms: uniform rows, rows of exact sigmoids 0, 1/2, 1)
 *   routing_map[t,e] = 1 for the k best probs of the token (ties -> lower e)
 *   tokens_per_expert[e] = sum_t routing_map[t,e]
 */
int oracle_aux_scores(int T, int E, int k, int score_fn, const float* logits, float* probs,
                      unsigned char* routing_map, int32_t* tokens_per_expert) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  int* sel = (int*)malloc(sizeof(int) * (size_t)k);
  for (int e = 0; e < E; ++e) tokens_per_expert[e] = 0;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    float* p = probs + (size_t)t * E;
    if (score_fn == ORC_SOFTMAX) {
      softmax_f32(l, E, p);
    } else {
      float s = 0.0f;
      for (int e = 0; e < E; ++e) {
        p[e] = sigmoid_f32(l[e]);
        s = s + p[e];
      }
      for (int e = 0; e < E; ++e) p[e] = p[e] / s;
    }
    pick_topk(p, NULL, E, k, sel);
    memset(routing_map + (size_t)t * E, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      routing_map[(size_t)t * E + sel[j]] = 1;
      tokens_per_expert[sel[j]] += 1;
    }
  }
  free(sel);
  return 0;
}

/*
 * Load-balancing loss [TE: Description, fused_moe_aux_loss; Signature lists
 * probs, tokens_per_expert, total_num_tokens, num_experts, topk, coeff]:
 *   L = coeff * E / (T_total * k) * sum_e ( sum_t probs[t,e] ) * tpe[e]
 * READING: this combination of the listed arguments is the one the aux-loss
 * workload states.  Column sums and the dot product in double, rounded once.
 */
int oracle_aux_loss_fwd(int T_rows, int T_total, int E, int k, float coeff, const float* probs,
                        const int32_t* tokens_per_expert, float* loss) {
  if (T_rows < 0 || T_total <= 0 || E <= 0 || k <= 0) return -1;
  double dot = 0.0;
  for (int e = 0; e < E; ++e) {
    double col = 0.0;
    for (int t = 0; t < T_rows; ++t) col += (double)probs[(size_t)t * E + e];
    dot += col * (double)tokens_per_expert[e];
  }
  double c = (double)coeff * (double)E / ((double)T_total * (double)k);
  *loss = (float)(c * dot);
  return 0;
}

/*
 * Backward of the loss [TE: Description, "both forward and backward"].
 *   C = coeff * E / (T_total * k); tokens_per_expert is a constant.
 *   grad_probs[t,e]  = grad_loss * C * tpe[e]
 *   grad_logits[t,e] = p[t,e] * (grad_probs[t,e] - sum_j p[t,j] * grad_probs[t,j])
 *                      (softmax backward; READING: the scores are the softmax)
 * All in double, rounded once.  Either output may be NULL.
 */
int oracle_aux_loss_bwd(int T_rows, int T_total, int E, int k, float coeff, float grad_loss,
                        const float* probs, const int32_t* tokens_per_expert, float* grad_probs,
                        float* grad_logits) {
  if (T_rows < 0 || T_total <= 0 || E <= 0 || k <= 0) return -1;
  double c = (double)coeff * (double)E / ((double)T_total * (double)k);
  double* gp = (double*)malloc(sizeof(double) * (size_t)E);
  for (int e = 0; e < E; ++e) gp[e] = (double)grad_loss * c * (double)tokens_per_expert[e];
  for (int t = 0; t < T_rows; ++t) {
    const float* p = probs + (size_t)t * E;
    double dot = 0.0;
    for (int e = 0; e < E; ++e) dot += (double)p[e] * gp[e];
    for (int e = 0; e < E; ++e) {
      if (grad_probs) grad_probs[(size_t)t * E + e] = (float)gp[e];
      if (grad_logits) grad_logits[(size_t)t * E + e] = (float)((double)p[e] * (gp[e] - dot));
    }
  }
  free(gp);
  return 0;
}

/*
 * Backward of the routed weights [TE: Description, FusedTopkScoreFunction /
 * fused_topk_with_score_function, forward and backward]: dL/dlogits given
 * dL/dweights for the selection ids (the selection and the bias carry no
 * gradient).  The forward, per token, with s_e = sigmoid(l_e) or p = softmax(l):
 *   v_j = s_{e_j}                         (SIGMOID)
 *   v_j = p_{e_j}                         (SOFTMAX, softmax before top-k)
 *   v_j = softmax over the k selected l   (SOFTMAX, top-k on logits first)
 *   w_j = scale * v_j / sum_i v_i (renormalize) or scale * v_j.
 * Backward, written out in double and rounded once:
 *   gv_i = scale * gw_i                                   (no renorm)
 *   gv_i = scale / S * (gw_i - sum_j gw_j v_j / S)         (renorm, S = sum v)
 *   SIGMOID:       gl_{e_j} += gv_j * v_j * (1 - v_j)
 *   SOFTMAX pre:   gl_e = p_e * (sum_{j: e_j = e} gv_j - sum_j v_j gv_j)
 *   SOFTMAX post:  gl_{e_j} = v_j * (gv_j - sum_i v_i gv_i)
 * other entries 0.
 */
int oracle_route_weights_bwd(int T, int E, int k, int score_fn, int pre, int renorm, float scale,
                             const float* logits, const int32_t* ids, const float* grad_w, float* grad_logits) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  double* v = (double*)malloc(sizeof(double) * (size_t)k);
  double* gv = (double*)malloc(sizeof(double) * (size_t)k);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  double* gl = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    const int32_t* id = ids + (size_t)t * k;
    const float* gw = grad_w + (size_t)t * k;
    for (int j = 0; j < k; ++j)
      if (id[j] < 0 || id[j] >= E) {
        free(v); free(gv); free(p); free(gl);
        return -1;
      }
    if (score_fn == ORC_SIGMOID) {
      for (int j = 0; j < k; ++j) v[j] = 1.0 / (1.0 + exp(-(double)l[id[j]]));
    } else if (pre) {
      double m = l[0];
      for (int e = 1; e < E; ++e) if (l[e] > m) m = l[e];
      double z = 0.0;
      for (int e = 0; e < E; ++e) { p[e] = exp((double)l[e] - m); z += p[e]; }
      for (int e = 0; e < E; ++e) p[e] /= z;
      for (int j = 0; j < k; ++j) v[j] = p[id[j]];
    } else {
      double m = l[id[0]];
      for (int j = 1; j < k; ++j) if (l[id[j]] > m) m = l[id[j]];
      double z = 0.0;
      for (int j = 0; j < k; ++j) { v[j] = exp((double)l[id[j]] - m); z += v[j]; }
      for (int j = 0; j < k; ++j) v[j] /= z;
    }
    if (renorm) {
      double S = 0.0, dot = 0.0;
      for (int j = 0; j < k; ++j) { S += v[j]; dot += (double)gw[j] * v[j]; }
      for (int j = 0; j < k; ++j) gv[j] = (double)scale / S * ((double)gw[j] - dot / S);
    } else {
      for (int j = 0; j < k; ++j) gv[j] = (double)scale * (double)gw[j];
    }
    for (int e = 0; e < E; ++e) gl[e] = 0.0;
    if (score_fn == ORC_SIGMOID) {
      for (int j = 0; j < k; ++j) gl[id[j]] += gv[j] * v[j] * (1.0 - v[j]);
    } else if (pre) {
      double d = 0.0;
      for (int j = 0; j < k; ++j) d += v[j] * gv[j];
      for (int j = 0; j < k; ++j) gl[id[j]] += gv[j];
      for (int e = 0; e < E; ++e) gl[e] = p[e] * (gl[e] - d);
    } else {
      double d = 0.0;
      for (int j = 0; j < k; ++j) d += v[j] * gv[j];
      for (int j = 0; j < k; ++j) gl[id[j]] = v[j] * (gv[j] - d);
    }
    for (int e = 0; e < E; ++e) grad_logits[(size_t)t * E + e] = (float)gl[e];
  }
  free(v); free(gv); free(p); free(gl);
  return 0;
}

/*
 * Backward of the aux scores [TE: Description, fused_compute_score_for_moe_aux_loss
 * forward and backward]: given dL/dprobs, dL/dlogits for the softmax scores
 * probs = softmax(logits) per row:
 *   grad_logits[t,e] = p[t,e] * (g[t,e] - sum_j p[t,j] * g[t,j])
 * (the softmax Jacobian, written out); the sum and the product in double,
 * rounded once.  score_fn SIGMOID: -2 (READING: the sigmoid scores normalised by
 * their row sum need that sum, which the probs alone do not give).
 */
int oracle_aux_scores_bwd(int T, int E, int score_fn, const float* probs, const float* grad_probs,
                          float* grad_logits) {
  if (T < 0 || E <= 0) return -1;
  if (score_fn != ORC_SOFTMAX) return -2;
  for (int t = 0; t < T; ++t) {
    const float* p = probs + (size_t)t * E;
    const float* g = grad_probs + (size_t)t * E;
    double dot = 0.0;
    for (int e = 0; e < E; ++e) dot += (double)p[e] * (double)g[e];
    for (int e = 0; e < E; ++e) grad_logits[(size_t)t * E + e] = (float)((double)p[e] * ((double)g[e] - dot));
  }
  return 0;
}

/*
 * Backward of the aux scores from the logits [TE: Description,
 * fused_compute_score_for_moe_aux_loss, "both forward and backward"; I/O
 * Contract, score_function "softmax" or "sigmoid"]: the vector-Jacobian
 * product of the forward's scores p(x) with the upstream gradient g, the
 * scores recomputed from the logits (READING: for sigmoid the scores are the
 * sigmoids divided by their row sum, as the forward states, so the row sum --
 * which the probs do not carry -- comes from the logits).
 *   softmax: p = softmax(x);          grad_i = p_i * (g_i - sum_e g_e p_e)
 *   sigmoid: s = sigmoid(x), S = sum s, p = s / S;
 *            dp_e/dx_i = s_i (1 - s_i) (delta_ei - p_e) / S
 *            grad_i = s_i (1 - s_i) / S * (g_i - sum_e g_e p_e)
 * All in double from the fp32 inputs, rounded once.
 */
int oracle_aux_scores_bwd_logits(int T, int E, int score_fn, const float* logits, const float* grad_probs,
                                 float* grad_logits) {
  if (T < 0 || E <= 0) return -1;
  if (score_fn != ORC_SOFTMAX && score_fn != ORC_SIGMOID) return -1;
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  double* d = (double*)malloc(sizeof(double) * (size_t)E);  /* dp_i/dx_i without the -p_i part */
  for (int t = 0; t < T; ++t) {
    const float* x = logits + (size_t)t * E;
    const float* g = grad_probs + (size_t)t * E;
    double sum = 0.0;
    if (score_fn == ORC_SOFTMAX) {
      double m = x[0];
      for (int e = 1; e < E; ++e) m = x[e] > m ? x[e] : m;
      for (int e = 0; e < E; ++e) {
        p[e] = exp((double)x[e] - m);
        sum += p[e];
      }
      for (int e = 0; e < E; ++e) {
        p[e] /= sum;
        d[e] = p[e];
      }
    } else {
      for (int e = 0; e < E; ++e) {
        p[e] = 1.0 / (1.0 + exp(-(double)x[e]));
        sum += p[e];
      }
      for (int e = 0; e < E; ++e) {
        d[e] = p[e] * (1.0 - p[e]) / sum;
        p[e] /= sum;
      }
    }
    double dot = 0.0;
    for (int e = 0; e < E; ++e) dot += (double)g[e] * p[e];
    for (int e = 0; e < E; ++e) grad_logits[(size_t)t * E + e] = (float)(d[e] * ((double)g[e] - dot));
  }
  free(p);
  free(d);
  return 0;
}

/*
 * Dispatch [LMD: invokeMoeDispatch]: copy each token's hidden row to each of
 * its k permuted rows; padding rows below P (p2t == -1) are zero (READING);
 * rows at or past P are left untouched.  Rows are raw 16-bit elements.
 */
int oracle_dispatch(int T, int H, int k, const uint16_t* hidden, const int32_t* e2p,
                    const int32_t* p2t, int32_t P, uint16_t* out) {
  if (T < 0 || H <= 0 || k <= 0 || P < 0) return -1;
  for (int32_t p = 0; p < P; ++p)
    if (p2t[p] < 0) memset(out + (size_t)p * H, 0, sizeof(uint16_t) * (size_t)H);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int32_t p = e2p[(size_t)t * k + j];
      if (p < 0) continue;
      memcpy(out + (size_t)p * H, hidden + (size_t)t * H, sizeof(uint16_t) * (size_t)H);
    }
  return 0;
}

/*
 * Combine [LMD: invokeMoeCombine, routing scales]: out[t,:] = bf16( the
 * fp32-accumulated weighted sum of the token's k expert rows ).  READING: the
 * accumulation is fp32 in slot order, acc = acc + w_j * x (a rounded product,
 * then a rounded add; no fused multiply-add), starting from 0, with the weights
 * read in their stored dtype; the sum is rounded once to bf16 (nearest even).
 * Slots with e2p < 0 contribute nothing.
 */
int oracle_combine(int T, int H, int k, const uint16_t* expert_out, const int32_t* e2p,
                   const void* weights, int weights_dtype, uint16_t* out) {
  if (T < 0 || H <= 0 || k <= 0) return -1;
  float* acc = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int h = 0; h < H; ++h) acc[h] = 0.0f;
    for (int j = 0; j < k; ++j) {
      int32_t p = e2p[(size_t)t * k + j];
      if (p < 0) continue;
      float w = load_elem(weights, weights_dtype, (size_t)t * k + j);
      const uint16_t* row = expert_out + (size_t)p * H;
      for (int h = 0; h < H; ++h) {
        float prod = w * bf16_to_f32(row[h]);
        acc[h] = acc[h] + prod;
      }
    }
    for (int h = 0; h < H; ++h) out[(size_t)t * H + h] = f32_to_bf16(acc[h]);
  }
  free(acc);
  return 0;
}

/*
 * Combine of fp32 expert rows into fp32 token rows [LMD: invokeMoeCombine,
 * routing scales]: the same READING as the bf16 combine (fp32 accumulation in
 * slot order, acc = acc + w_j * x with a rounded product and a rounded add,
 * starting from 0; weights in their stored dtype; slots with e2p < 0 skipped),
 * and the fp32 sum is the result (no further rounding).
 */
int oracle_combine_f32(int T, int H, int k, const float* expert_out, const int32_t* e2p,
                       const void* weights, int weights_dtype, float* out) {
  if (T < 0 || H <= 0 || k <= 0) return -1;
  for (int t = 0; t < T; ++t) {
    float* acc = out + (size_t)t * H;
    for (int h = 0; h < H; ++h) acc[h] = 0.0f;
    for (int j = 0; j < k; ++j) {
      int32_t p = e2p[(size_t)t * k + j];
      if (p < 0) continue;
      float w = load_elem(weights, weights_dtype, (size_t)t * k + j);
      const float* row = expert_out + (size_t)p * H;
      for (int h = 0; h < H; ++h) {
        float prod = w * row[h];
        acc[h] = acc[h] + prod;
      }
    }
  }
  return 0;
}

/*
 * Expert-parallel regroup [NKI: Background, the all-to-all-v MoE dispatch
 * path; TRT: Parameters local_expert_offset / local_num_experts, Returns].
 * counts[s*L + e]: rows rank s sends for this rank's local expert e; recv
 * holds them ordered by source, then expert, then the source's token order.
 * READING: the receiving rank lays its rows out by local expert, then source
 * rank, then token (the order a single route of all ranks' tokens,
 * concatenated in rank order, gives), each expert padded to `tile` rows
 * (padding rows zero), padded_to_recv = the receive row of each padded row
 * (-1 on padding).  Rows are `row_bytes` bytes, copied as they are.
 */
int oracle_ep_regroup(int W, int L, int tile, const int32_t* counts, const uint8_t* recv, long long n_recv,
                      long long row_bytes, uint8_t* padded, int32_t* offsets, int32_t* totals,
                      int32_t* padded_to_recv) {
  if (W <= 0 || L <= 0 || tile <= 0 || row_bytes <= 0) return -1;
  long long n = 0;
  for (int i = 0; i < W * L; ++i) {
    if (counts[i] < 0) return -1;
    n += counts[i];
  }
  if (n != n_recv) return -1;
  offsets[0] = 0;
  for (int e = 0; e < L; ++e) {
    int tot = 0;
    for (int s = 0; s < W; ++s) tot += counts[s * L + e];
    offsets[e + 1] = offsets[e] + (tot + tile - 1) / tile * tile;
  }
  int P = offsets[L];
  for (int p = 0; p < P; ++p) {
    padded_to_recv[p] = -1;
    memset(padded + (size_t)p * row_bytes, 0, (size_t)row_bytes);
  }
  long long r = 0;
  for (int s = 0; s < W; ++s) {
    for (int e = 0; e < L; ++e) {
      int before = 0;  /* rows of expert e from earlier sources */
      for (int s2 = 0; s2 < s; ++s2) before += counts[s2 * L + e];
      for (int i = 0; i < counts[s * L + e]; ++i, ++r) {
        int p = offsets[e] + before + i;
        memcpy(padded + (size_t)p * row_bytes, recv + (size_t)r * row_bytes, (size_t)row_bytes);
        padded_to_recv[p] = (int32_t)r;
      }
    }
  }
  totals[0] = P;
  totals[1] = P / tile;
  return 0;
}

/*
 * Fused RMSNorm + router + top-k for small decode batches [NKI: Background;
 * Parameters; Returns; Notes].
 *   r_t       = 1 / sqrt( mean_h x[t,h]^2 + eps )                 (double)
 *   xn[t,h]   = bf16( x[t,h] * r_t * gamma[h] )                     (double, one rounding)
 *   logit[t,e]= fp32( sum_h xn[t,h] * W[h,e] + b[e] )               (double, one rounding)
 *               READING: the projection consumes the stored bf16 xn
 *   ids       = top-k on the raw logits (ACT2: activation after top-k),
 *               (logit desc, expert asc)
 *   aff[t,e]  = bf16( sigmoid(logit) ) at the selected experts (fp32 formula),
 *               or, for SOFTMAX, bf16 of the softmax over the k selected
 *               logits; 0 elsewhere
 * Constraints [NKI: Notes]: T <= 128, H % 128 == 0.
 */
int oracle_rmsnorm_router_topk(int T, int H, int E, int k, float eps, int act,
                               const uint16_t* hidden, const uint16_t* gamma, const uint16_t* W,
                               const uint16_t* bias, uint16_t* out_norm, int32_t* ids,
                               uint16_t* aff, float* logits_out) {
  if (T < 0 || T > 128 || H <= 0 || H % 128 != 0 || E <= 0 || k <= 0 || k > E) return -1;
  float* lg = (float*)malloc(sizeof(float) * (size_t)E);
  float* xnf = (float*)malloc(sizeof(float) * (size_t)H);
  int* sel = (int*)malloc(sizeof(int) * (size_t)k);
  float* v = (float*)malloc(sizeof(float) * (size_t)k);
  for (int t = 0; t < T; ++t) {
    const uint16_t* x = hidden + (size_t)t * H;
    double ss = 0.0;
    for (int h = 0; h < H; ++h) {
      double xv = (double)bf16_to_f32(x[h]);
      ss += xv * xv;
    }
    double r = 1.0 / sqrt(ss / (double)H + (double)eps);
    for (int h = 0; h < H; ++h) {
      double y = (double)bf16_to_f32(x[h]) * r * (double)bf16_to_f32(gamma[h]);
      uint16_t q = f64_to_bf16(y);
      out_norm[(size_t)t * H + h] = q;
      xnf[h] = bf16_to_f32(q);
    }
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h) acc += (double)xnf[h] * (double)bf16_to_f32(W[(size_t)h * E + e]);
      if (bias) acc += (double)bf16_to_f32(bias[e]);
      lg[e] = (float)acc;
    }
    if (logits_out) memcpy(logits_out + (size_t)t * E, lg, sizeof(float) * (size_t)E);
    pick_topk(lg, NULL, E, k, sel);
    if (act == ORC_SOFTMAX) {
      float* sl = (float*)malloc(sizeof(float) * (size_t)k);
      for (int j = 0; j < k; ++j) sl[j] = lg[sel[j]];
      softmax_f32(sl, k, v);
      free(sl);
    } else {
      for (int j = 0; j < k; ++j) v[j] = sigmoid_f32(lg[sel[j]]);
    }
    for (int e = 0; e < E; ++e) aff[(size_t)t * E + e] = 0;
    for (int j = 0; j < k; ++j) {
      ids[(size_t)t * k + j] = sel[j];
      aff[(size_t)t * E + sel[j]] = f32_to_bf16(v[j]);
    }
  }
  free(lg); free(xnf); free(sel); free(v);
  return 0;
}

/*
 * Router projection alone [NKI: Parameters, router_weights [H,E], router_bias]:
 * logit[t,e] = fp32( sum_h xn[t,h] * W[h,e] + b[e] ), double accumulation, one
 * rounding; xn given as bf16 (lets a test isolate the projection from the
 * normalisation).
 */
int oracle_router_logits(int T, int H, int E, const uint16_t* xn, const uint16_t* W, const uint16_t* bias,
                         float* logits) {
  if (T < 0 || H <= 0 || E <= 0) return -1;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)bf16_to_f32(xn[(size_t)t * H + h]) * (double)bf16_to_f32(W[(size_t)h * E + e]);
      if (bias) acc += (double)bf16_to_f32(bias[e]);
      logits[(size_t)t * E + e] = (float)acc;
    }
  return 0;
}
