// moe_route: expert selection, routing weights and permutation bookkeeping in
// two launches chained by programmatic dependent launch.
//
// Sources (by page title and section):
//   Implementation:NVIDIA TransformerEngine Fused Router -- Description
//     (fused_topk_with_score_function: score function, pre/post softmax, group
//     top-k and expert bias in one kernel), I/O Contract;
//   flashinfer.fused_moe.trtllm_gen_routing -- Parameters, Returns, Notes
//     (permutation outputs, tile padding, tile -> expert identity);
//   max.nn.moe.SigmoidTopKRouter -- steps 2-4 (sigmoid, select on score +
//     correction bias, weight by the unbiased score, renormalise, scale);
//   Implementation:InternLM Lmdeploy Gemm MoeUtils -- invokeMoeGate_V2 (maps
//     and per-expert offsets).
//
// The tokens are split into G contiguous segments of at most B tokens; block c
// of both kernels owns segment c.
//
// route_select_kernel (one block per segment)
//   Each token is scored and its top-k selected; ids and weights are written.
//   Every selection also sets bit lt (the token's index in the segment) in a
//   shared-memory bitmask of its expert.  After the block's selections, the
//   rank of selection (t, e) among the segment's selections of e in token
//   order is the number of bits of e's mask below lt (popcounts), and e's
//   count is the number of all its bits.  The block writes the counts as its
//   row of a table in the workspace and parks (expert, rank) of every
//   selection in expanded_to_permuted.  Selection paths:
//     - sigmoid fast path (E = 8*V): 8 lanes per token, a lane per V experts
//       (one expert group when n_group = 8), 4 tokens per warp; each warp
//       stages its 4 token rows in shared memory with one bulk copy (TMA),
//       double-buffered.  A proxy key from tanh.approx (error <= delta)
//       bounds where the exact keys can matter: exact fp32 keys (the stated
//       formula) are computed only for each lane's top-2 region (exact group
//       scores) and for the candidates of the top-k, which are ranked by
//       counting.  A token whose candidates overflow falls back to exact keys
//       for all its experts;
//     - generic: a warp per token (E > 32) or a thread per token (E <= 32)
//       with exact keys and k rounds of argmax, logits read from global memory.
//   The segments form groups of GS consecutive segments; each selection block
//   also adds its counts into its group's row of per-group totals (integer
//   atomics: order-free, so the totals are deterministic).
// route_permute_kernel (one block per segment, launched as the dependent)
//   Every block adds the group totals (the expert counts; those of the groups
//   before its own plus the table rows of its group's earlier segments give its
//   base per expert), scans the tile-padded offsets, and turns each parked
//   (expert, rank) into the slot offset + base + rank (deterministic, token
//   order); it also writes its share of the tile tables and of the padding
//   rows of permuted_to_token.  The last block to have read the group totals
//   (a ticket) clears them for the next call.
// Neither kernel waits on another block, so no device-side wait can time out
// (the only bounded waits are on the block's own bulk copies).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace moe {

namespace {

constexpr int kFastWarpsMax = 28;        // fast path: up to 28 warps of 4 tokens (72 registers a thread)
constexpr int kGenericThreads = 512;     // generic paths
constexpr int kPermThreads = 1024;       // bookkeeping kernel
constexpr int kMaxSegment = 256;         // tokens per segment (8 mask words)
constexpr int kMaxGroups = 16;           // segment groups whose count totals the selection accumulates

struct RouteArgs {
  const void* logits;
  const void* bias;
  int32_t* ids;
  void* weights;
  int32_t* counts;
  int32_t* offsets;
  int32_t* e2p;
  int32_t* p2t;
  int32_t* tile_expert;
  int32_t* tile_mn;
  int32_t* totals;
  WsHeader* hdr;
  uint8_t* table;    // [G][row_stride]: per-segment expert counts (cnt_bytes wide)
  uint32_t* gtot;    // [NG][E]: per-group expert counts (groups of GS segments), zero between calls
  int T, E, k;
  int S, kt, E2;     // fused shared experts (ids E .. E+S-1), slots per token k + S, experts counted E + S
  int score_fn, pre, grouped, n_group, topk_group, topn;
  int renorm;
  float scale;
  int tile;          // power of two
  uint32_t kinv;     // ceil(2^32 / kt): item -> token by a multiply-high
  int logits_dtype, bias_dtype, weights_dtype;
  int has_bias;
  int G, B;          // segments, tokens per segment (segment c: [c*B, min(T, (c+1)*B)))
  int MW;            // 32-bit mask words per expert: ceil(B / 32)
  int GS, NG;        // segments per group, groups
  int slots;         // fast path: staging slots per warp (1 when every warp has one quad, else 2)
  int max_padded;
  int max_tiles;
  int loc_off, loc_n;  // the local experts [loc_off, loc_off + loc_n): only they get slots and tiles
  int row_bytes;     // bytes per logits row
  int cnt_bytes;     // width of a table entry: 1 (B <= 255) or 2
  int row_stride;    // bytes per table row (16-byte multiple)
  long long timeout_ns;
};

// ---------------------------------------------------------------------------
// shared-memory layout of the selection kernel
// ---------------------------------------------------------------------------
struct SelSmem {
  int masks, ids, bias, cb, delta, warp0, warp_bytes, total;
  int stage_bytes;  // per staging slot (fast path)
};

constexpr int kCandSlotsPerToken = 32;  // fast path: candidates ranked per token
// fast path: a warp's tokens left to the exact path; a segment holds at most
// 256 tokens = 64 quads over at least 28 warps (or one quad per warp), so a
// warp runs at most 3 rounds of 4 tokens
constexpr int kPendMax = 12;
constexpr int kCandBytes = 4 * kCandSlotsPerToken * 14 + 2 * kPendMax + 8;

// per warp (fast path): 2 staging slots of 4 rows; 4 tokens x 32 packed u64
// candidate keys, 4 x 32 fp32 scores and 4 x 32 u16 expert ids; the warp's
// pending exact-path tokens; 2 mbarriers
__host__ __device__ inline SelSmem sel_smem_layout(int E, int MW, int B, int k, int fast, int V, int row_bytes,
                                                   int nwarps, int slots) {
  SelSmem L;
  int o = 0;
  L.masks = o;
  o += ((E * MW * 4) + 15) & ~15;  // every region starts on 16 bytes (the constants are read as 16-byte vectors)
  L.ids = o;
  o += ((B * k * 2) + 15) & ~15;
  L.bias = o;
  o += ((E * 4) + 15) & ~15;
  L.cb = o;  // fast path: 8 rows of V f16 constants 0.5 + b, 16 bytes of padding each
  o += fast ? 8 * (V * 2 + 16) : 0;
  L.delta = o;  // fast path: the block's proxy error bound
  o += fast ? 16 : 0;
  o = (o + 127) & ~127;
  L.warp0 = o;
  L.stage_bytes = fast ? ((4 * row_bytes + 127) & ~127) : 0;
  L.warp_bytes = fast ? ((slots * L.stage_bytes + kCandBytes + 16 + 127) & ~127) : 0;
  o += L.warp_bytes * nwarps;
  L.total = o;
  return L;
}

__device__ __forceinline__ float stage_val(const RouteArgs& a, const uint8_t* row, int e) {
  if (a.logits_dtype == MOE_BF16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(row)[e]);
  return reinterpret_cast<const float*>(row)[e];
}

__device__ __forceinline__ float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

// expert e belongs to this shard: it gets rows, slots and tiles (a fused
// shared expert, e >= E, is local on every shard)
__device__ __forceinline__ bool is_local(const RouteArgs& a, int e) {
  return (unsigned)(e - a.loc_off) < (unsigned)a.loc_n || e >= a.E;
}
// the local index of a local expert: the shard's routed experts, then the shared ones
__device__ __forceinline__ int local_index(const RouteArgs& a, int e) {
  return e >= a.E ? a.loc_n + (e - a.E) : e - a.loc_off;
}

// One selection of expert e by the segment's token lt at slot j: the id in the
// segment's list, the token's bit in e's mask.
__device__ __forceinline__ void mark(const RouteArgs& a, uint32_t* masks, uint16_t* ids_s, int lt, int j, int e) {
  ids_s[lt * a.kt + j] = (uint16_t)e;
  atomicOr(&masks[e * a.MW + (lt >> 5)], 1u << (lt & 31));
}

// -------------------------------------------------------------------------
// warp per token (E > 32): lane l owns experts [l*VPL, l*VPL + VPL)
// -------------------------------------------------------------------------
template <int VPL>
__device__ void select_token_warp(const RouteArgs& a, const uint8_t* row, long long t, int lt, const float* bias_s,
                                  uint32_t* masks, uint16_t* ids_s, int lane) {
  const int E = a.E;
  const unsigned FULL = 0xffffffffu;
  float lg[VPL], s[VPL], key[VPL];
  uint32_t valid = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane * VPL + i;
    const bool v = e < E;
    lg[i] = v ? stage_val(a, row, e) : 0.0f;
    valid |= (v ? 1u : 0u) << i;
  }
  // ---- score ----
  if (!a.pre) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) s[i] = lg[i];
  } else if (a.score_fn == MOE_SOFTMAX) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (valid & (1u << i)) m = fmaxf(m, lg[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      s[i] = (valid & (1u << i)) ? expf(lg[i] - m) : 0.0f;
      sum += s[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
#pragma unroll
    for (int i = 0; i < VPL; ++i) s[i] = s[i] / sum;
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) s[i] = sigmoid_f32(lg[i]);
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane * VPL + i;
    key[i] = s[i] + ((a.has_bias && e < E) ? bias_s[e] : 0.0f);
  }
  uint32_t allowed = valid;

  // ---- groups ----
  if (a.grouped) {
    const int GS = E / a.n_group;
    if (GS >= VPL) {
      // a group spans LG = GS / VPL lanes (a power of two, checked on the host)
      const int LG = GS / VPL;
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        if (valid & (1u << i)) {
          const float x = key[i];
          const float hi = fmaxf(m1, x);
          m2 = fmaxf(m2, fminf(m1, x));
          m1 = hi;
        }
      }
      for (int off = 1; off < LG; off <<= 1) {
        const float o1 = __shfl_xor_sync(FULL, m1, off);
        const float o2 = __shfl_xor_sync(FULL, m2, off);
        const float hi = fmaxf(m1, o1);
        m2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = hi;
      }
      const float gsc = (a.topn == 1) ? m1 : (m1 + m2);
      const int myg = lane / LG;
      int rank = 0;
      for (int g = 0; g < a.n_group; ++g) {
        const float o = __shfl_sync(FULL, gsc, (g * LG) & 31);
        rank += (o > gsc || (o == gsc && g < myg)) ? 1 : 0;
      }
      if (lane * VPL >= E || rank >= a.topk_group) allowed = 0;
    } else {
      // a lane holds NG = VPL / GS whole groups
      const int NG = VPL / GS;
      float mygsc[VPL];
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        if (q < NG) {
          float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            if (i / GS == q && (valid & (1u << i))) {
              const float x = key[i];
              const float hi = fmaxf(m1, x);
              m2 = fmaxf(m2, fminf(m1, x));
              m1 = hi;
            }
          }
          mygsc[q] = (a.topn == 1) ? m1 : (m1 + m2);
        }
      }
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        if (q < NG) {
          const int myg = lane * NG + q;
          int rank = 0;
          for (int g = 0; g < a.n_group; ++g) {
            // fetch group g's score from lane g / NG, slot g % NG
            float cand = 0.0f;
#pragma unroll
            for (int r = 0; r < VPL; ++r)
              if (r < NG && r == g % NG) cand = mygsc[r];
            const float o = __shfl_sync(FULL, cand, (g / NG) & 31);
            rank += (o > mygsc[q] || (o == mygsc[q] && g < myg)) ? 1 : 0;
          }
          if (myg >= a.n_group || rank >= a.topk_group) {
#pragma unroll
            for (int i = 0; i < VPL; ++i)
              if (i / GS == q) allowed &= ~(1u << i);
          }
        }
      }
    }
  }

  // ---- top-k: k rounds of warp argmax over packed (key, ~expert) ----
  int my_id = 0;
  float my_v = 0.0f;
  for (int j = 0; j < a.k; ++j) {
    unsigned long long best = 0ull;
    float best_s = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (allowed & (1u << i)) {
        const unsigned long long pk = pack_key(key[i], lane * VPL + i);
        if (pk > best) {
          best = pk;
          best_s = s[i];
        }
      }
    }
    unsigned long long wbest = best;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const unsigned long long o = shfl_xor_u64(FULL, wbest, off);
      wbest = o > wbest ? o : wbest;
    }
    const int win = packed_expert(wbest);
    const int owner = win / VPL;
    const float win_s = __shfl_sync(FULL, best_s, owner);
    if (lane == owner) allowed &= ~(1u << (win - owner * VPL));
    if (lane == j) {
      my_id = win;
      my_v = win_s;
    }
  }

  // ---- weights (lanes < k hold slot j = lane) ----
  const bool has_slot = lane < a.k;
  float v = my_v;
  if (!a.pre) {
    if (a.score_fn == MOE_SOFTMAX) {
      float m = has_slot ? v : -INFINITY;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
      float ex = has_slot ? expf(v - m) : 0.0f;
      float sum = ex;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
      v = ex / sum;
    } else {
      v = sigmoid_f32(v);
    }
  }
  if (a.renorm) {
    float sum = has_slot ? v : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
    v = (v / sum) * a.scale;
  } else {
    v = v * a.scale;
  }
  if (has_slot) {
    const size_t o = (size_t)t * a.kt + lane;
    a.ids[o] = my_id;
    store_from_f32(a.weights, a.weights_dtype, o, v);
    if ((unsigned)my_id < (unsigned)E) mark(a, masks, ids_s, lt, lane, my_id); else record_bounds(a.hdr);
  }
}

// -------------------------------------------------------------------------
// thread per token (E <= EMAX <= 32)
// -------------------------------------------------------------------------
template <int EMAX>
__device__ void select_token_thread(const RouteArgs& a, const uint8_t* row, long long t, int lt, const float* bias_s,
                                    uint32_t* masks, uint16_t* ids_s) {
  const int E = a.E;
  float lg[EMAX], s[EMAX], key[EMAX];
#pragma unroll
  for (int i = 0; i < EMAX; ++i) lg[i] = (i < E) ? stage_val(a, row, i) : 0.0f;
  if (!a.pre) {
#pragma unroll
    for (int i = 0; i < EMAX; ++i) s[i] = lg[i];
  } else if (a.score_fn == MOE_SOFTMAX) {
    float m = lg[0];
#pragma unroll
    for (int i = 1; i < EMAX; ++i)
      if (i < E && lg[i] > m) m = lg[i];
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < EMAX; ++i) {
      s[i] = (i < E) ? expf(lg[i] - m) : 0.0f;
      sum = sum + s[i];
    }
#pragma unroll
    for (int i = 0; i < EMAX; ++i) s[i] = s[i] / sum;
  } else {
#pragma unroll
    for (int i = 0; i < EMAX; ++i) s[i] = sigmoid_f32(lg[i]);
  }
#pragma unroll
  for (int i = 0; i < EMAX; ++i) key[i] = s[i] + ((a.has_bias && i < E) ? bias_s[i] : 0.0f);
  uint32_t allowed = (E >= 32) ? 0xffffffffu : ((1u << E) - 1u);

  if (a.grouped) {
    const int GS = E / a.n_group;
    float gsc[EMAX];
    for (int g = 0; g < a.n_group; ++g) {
      float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
      for (int i = 0; i < EMAX; ++i) {
        if (i >= g * GS && i < (g + 1) * GS) {
          const float x = key[i];
          const float hi = fmaxf(m1, x);
          m2 = fmaxf(m2, fminf(m1, x));
          m1 = hi;
        }
      }
      gsc[g] = (a.topn == 1) ? m1 : (m1 + m2);
    }
    for (int g = 0; g < a.n_group; ++g) {
      int rank = 0;
      for (int h = 0; h < a.n_group; ++h) rank += (gsc[h] > gsc[g] || (gsc[h] == gsc[g] && h < g)) ? 1 : 0;
      if (rank >= a.topk_group) {
#pragma unroll
        for (int i = 0; i < EMAX; ++i)
          if (i >= g * GS && i < (g + 1) * GS) allowed &= ~(1u << i);
      }
    }
  }

  int sel[EMAX];
  float val[EMAX];
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    sel[j] = 0;
    val[j] = 0.0f;
    if (j < a.k) {
      int b = -1;
      float bk = 0.0f, bs = 0.0f;
#pragma unroll
      for (int i = 0; i < EMAX; ++i) {
        if ((allowed >> i) & 1u) {
          if (b < 0 || key[i] > bk) {
            b = i;
            bk = key[i];
            bs = s[i];
          }
        }
      }
      allowed &= ~(1u << b);
      sel[j] = b;
      val[j] = bs;
    }
  }
  if (!a.pre) {
    if (a.score_fn == MOE_SOFTMAX) {
      float m = val[0];
#pragma unroll
      for (int j = 1; j < EMAX; ++j)
        if (j < a.k && val[j] > m) m = val[j];
      float sum = 0.0f;
#pragma unroll
      for (int j = 0; j < EMAX; ++j) {
        if (j < a.k) {
          val[j] = expf(val[j] - m);
          sum = sum + val[j];
        }
      }
#pragma unroll
      for (int j = 0; j < EMAX; ++j)
        if (j < a.k) val[j] = val[j] / sum;
    } else {
#pragma unroll
      for (int j = 0; j < EMAX; ++j)
        if (j < a.k) val[j] = sigmoid_f32(val[j]);
    }
  }
  float norm = 1.0f;
  if (a.renorm) {
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < EMAX; ++j)
      if (j < a.k) sum = sum + val[j];
    norm = sum;
  }
#pragma unroll
  for (int j = 0; j < EMAX; ++j) {
    if (j < a.k) {
      const float w = a.renorm ? (val[j] / norm) * a.scale : val[j] * a.scale;
      const size_t o = (size_t)t * a.kt + j;
      a.ids[o] = sel[j];
      store_from_f32(a.weights, a.weights_dtype, o, w);
      if ((unsigned)sel[j] < (unsigned)E) mark(a, masks, ids_s, lt, j, sel[j]); else record_bounds(a.hdr);
    }
  }
}

// -------------------------------------------------------------------------
// sigmoid fast path: 8 lanes per token, lane g owns experts [g*V, (g+1)*V)
// -------------------------------------------------------------------------
// The proxy key of the fast path, two experts at a time in half precision:
//   p = 0.5 * tanh.approx(x / 2) + (0.5 + b)   (sigmoid(x) = 0.5 + 0.5 tanh(x/2))
// with x rounded to f16 (exact for bf16 logits in the f16 range), the tanh and
// the fused multiply-add in packed f16.  cb2 holds 0.5 + b of both experts in
// f16.  |p - (sigmoid(x) + b)| <= proxy_delta(...) (see below).
__device__ __forceinline__ __half2 proxy_pair(float xlo, float xhi, __half2 cb2) {
  const __half2 half = __float2half2_rn(0.5f);
  const __half2 h = __hmul2(__floats2half2_rn(xlo, xhi), half);
  return __hfma2(h2tanh_approx(h), half, cb2);
}

// Absolute error bound of proxy_pair over a block whose experts have
// |0.5 + b| <= cbmax: half the assumed tanh.approx.f16 error (|t| <= 1), the
// f16 rounding of 0.5 + b and of the fused multiply-add's result (|p| <= 0.5 +
// cbmax), the f16 rounding of fp32 logits (|sigmoid'(x) x| <= 0.224, i.e.
// <= 2^-13 at 11 bits), and slack for the fp32 sigmoid's own rounding.
// kTanh16Err is checked against every f16 input by the test suite, and the
// whole bound against every bf16 logit under a sweep of biases.
constexpr float kTanh16Err = 1.0f / 1024.0f;
__host__ __device__ inline float half_ulp16(float v) {
  // half an f16 ulp at magnitude v (v >= 2^-14): 2^(floor(log2 v) - 11)
  int e = 0;
  float m = v;
  while (m >= 2.0f) { m *= 0.5f; ++e; }
  while (m < 1.0f && e > -14) { m *= 2.0f; --e; }
  float r = 1.0f;
  for (int i = 0; i < 11 - e; ++i) r *= 0.5f;
  for (int i = 0; i < e - 11; ++i) r *= 2.0f;
  return r;
}
__host__ __device__ inline float proxy_delta(float cbmax, int f32_logits) {
  if (!(cbmax <= 1024.0f)) return INFINITY;  // f16 too coarse: every expert becomes a candidate
  const float d = 0.5f * kTanh16Err + half_ulp16(cbmax) + half_ulp16(0.5f + cbmax) +
                  (f32_logits ? 1.0f / 8192.0f : 0.0f) + 1.0f / (1 << 20);
  return d;
}

// A lane reads its NC 16-byte chunks starting at chunk `rot` = g*NC/8, so the 8
// lanes of a token hit distinct bank groups (its rows are contiguous in shared
// memory).  Register slot j then holds this expert:
template <int V, int ESZ>
__device__ __forceinline__ int slot_expert(int g, int rot, int j) {
  constexpr int EPC = 16 / ESZ, NC = V / EPC;
  return g * V + (((j / EPC) + rot) & (NC - 1)) * EPC + (j % EPC);
}
template <int V, int ESZ>
__device__ __forceinline__ int expert_slot(int g, int rot, int e) {
  constexpr int EPC = 16 / ESZ, NC = V / EPC;
  const int r = e - g * V;
  return (((r / EPC) - rot + NC) & (NC - 1)) * EPC + (r % EPC);
}

// Per-lane constants 0.5 + bias of the lane's experts in f16, in register-slot
// order: one row of V halves + 16 bytes of padding per lane position g (the
// 16-byte loads of the 8 lanes of a token fall in distinct bank groups).
template <int V>
__host__ __device__ constexpr int cb_stride_bytes() { return V * 2 + 16; }

// Bits of a packed mask: pair i's low half (slot 2i) is bit i, its high half
// (slot 2i+1) bit 16 + i.
__device__ __forceinline__ int mask_bit_slot(int b) { return b < 16 ? 2 * b : 2 * (b - 16) + 1; }

// Mask of the lane's slots whose proxy is >= thr (thr rounded down to f16).
template <int NW>
__device__ __forceinline__ uint32_t proxy_mask(const __half2 (&p2)[NW], float thr) {
  const __half t = __float2half_rd(thr);
  const __half2 t2 = __halves2half2(t, t);
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) m |= (__hge2_mask(p2[i], t2) >> (15 - i)) & (0x00010001u << i);
  return m;
}

constexpr int kCandSlots = kCandSlotsPerToken;  // more candidates send the token to the exact path

// One quad of tokens (lane = 8*q + g: token q, experts of lane position g),
// their rows staged in shared memory at `rows`.  cand: per token kCandSlots
// packed (ordered key, ~expert) words, then kCandSlots fp32 scores.  Returns
// the mask of the quad's tokens left to the exact path (bit q).
//
// 1. Proxy keys p (|p - key| <= delta) of the lane's V experts and the lane's
//    top-2 proxies m1 >= m2 (the two largest keys lie within delta of them).
// 2. Groups (lane g = group g): the approximate group scores s = m1 + m2 (or
//    m1) are within e = 2 delta (delta) of the exact ones.  A group is surely
//    kept when fewer than topk_group others may reach its score (s_h + e >=
//    s_g - e), surely dropped when topk_group others surely beat it (s_h - e >
//    s_g + e); the others are undecided and stay candidates' sources until
//    their exact scores are known.
// 3. Threshold: each group that can be kept holds two experts with keys >=
//    its m2 - delta, and the kept groups hold 2 * topk_group >= k such
//    experts, so the k-th largest key is >= min m2 - delta over the groups
//    that can be kept (for ungrouped routing: the k-th largest of the lanes'
//    m1, m2, minus delta); an expert that can be in the top-k has a proxy >=
//    that minus delta.
// 4. Candidates (experts of the groups that can be kept, over the threshold;
//    at most kCandSlots per token): listed per token, their exact keys (the
//    stated formula) computed by the token's 8 lanes.  The threshold is below every such group's m2 - 2 delta,
//    so each undecided group's exact top-2 keys are candidates: its exact
//    score comes from its candidates, the undecided groups are ranked
//    exactly (ties -> lower group) and the dropped ones' candidates are
//    zeroed.  The candidates are ranked by counting on packed (ordered key,
//    ~expert) words: larger key first, then lower expert.
template <int V, int ESZ>
__device__ unsigned select_quad_fast(const RouteArgs& a, const uint8_t* rows, int lt0, int nq, long long t_seg,
                                     const uint8_t* cb_s, const float* bias_s, float delta, uint8_t* cand,
                                     uint32_t* masks, uint16_t* ids_s, int lane) {
  constexpr int EPC = 16 / ESZ, NC = V / EPC, NW = V / 2, PPC = EPC / 2;  // pairs per chunk
  const unsigned FULL = 0xffffffffu;
  const int q = lane >> 3, g = lane & 7, seg = lane & 24;
  const int rot = (g * NC) >> 3;
  const bool tv = q < nq;
  const uint8_t* row = rows + (size_t)(tv ? q : 0) * a.row_bytes;
  const int lt = lt0 + q;
  const long long t = t_seg + lt;
  unsigned long long* ck = reinterpret_cast<unsigned long long*>(cand) + q * kCandSlots;
  float* cs = reinterpret_cast<float*>(cand + 4 * kCandSlots * 8) + q * kCandSlots;

  // ---- 1. proxies, packed two per register, and their top-2 (two streams:
  //         even and odd slots) ----
  __half2 p2[NW];
  __half2 m1 = __float2half2_rn(-INFINITY), m2 = m1;
  const uint8_t* cbl = cb_s + g * cb_stride_bytes<V>();
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int cc = (c + rot) & (NC - 1);
    const uint4 v = *reinterpret_cast<const uint4*>(row + (size_t)g * V * ESZ + cc * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t cbw[4];
    if constexpr (PPC == 4) {
      const uint4 c4 = *reinterpret_cast<const uint4*>(cbl + c * 16);
      cbw[0] = c4.x; cbw[1] = c4.y; cbw[2] = c4.z; cbw[3] = c4.w;
    } else {
      const uint2 c2 = *reinterpret_cast<const uint2*>(cbl + c * 8);
      cbw[0] = c2.x; cbw[1] = c2.y;
    }
#pragma unroll
    for (int i = 0; i < PPC; ++i) {
      float xlo, xhi;
      if constexpr (ESZ == 2) {
        xlo = __uint_as_float(w[i] << 16);
        xhi = __uint_as_float(w[i] & 0xffff0000u);
      } else {
        xlo = __uint_as_float(w[2 * i]);
        xhi = __uint_as_float(w[2 * i + 1]);
      }
      const __half2 p = proxy_pair(xlo, xhi, *reinterpret_cast<const __half2*>(&cbw[i]));
      p2[c * PPC + i] = p;
      const __half2 hi = __hmax2(m1, p);
      m2 = __hmax2(m2, __hmin2(m1, p));
      m1 = hi;
    }
  }
  float M1, M2;
  {
    const float a1 = __low2float(m1), b1 = __high2float(m1), a2 = __low2float(m2), b2 = __high2float(m2);
    M1 = fmaxf(a1, b1);
    M2 = fmaxf(fminf(a1, b1), fmaxf(a2, b2));
  }

  // ---- 2. groups: surely kept, surely dropped, undecided ----
  bool maybe = true;   // this group can be kept
  bool undec = false;  // undecided: kept or not is settled by exact scores
  int K = 8;           // groups kept
  if (a.grouped) {
    K = a.topk_group;
    const float gsc = (a.topn == 1) ? M1 : (M1 + M2);
    const float e2 = (a.topn == 1 ? 2.0f : 4.0f) * delta;  // twice the score error
    int may_beat = 0, beats = 0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float o = __shfl_sync(FULL, gsc, seg | h);
      may_beat += (h != g && o + e2 >= gsc) ? 1 : 0;
      beats += (o - e2 > gsc) ? 1 : 0;
    }
    const bool sure = may_beat < K;
    maybe = beats < K;
    undec = maybe && !sure;
  }

  // ---- 3. candidate threshold ----
  float kth;
  if (a.grouped) {
    // min m2 over the groups that can be kept (2 * topk_group >= k on this path)
    float mn = maybe ? M2 : INFINITY;
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, 1));
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, 2));
    kth = fminf(mn, __shfl_xor_sync(FULL, mn, 4));
  } else {
    // the k-th largest of the 16 proxies m1, m2 of the token's lanes
    int gt1 = 0, ge1 = 0, gt2 = 0, ge2 = 0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float o1 = __shfl_sync(FULL, M1, seg | h), o2 = __shfl_sync(FULL, M2, seg | h);
      gt1 += (o1 > M1) + (o2 > M1);
      ge1 += (o1 >= M1) + (o2 >= M1);
      gt2 += (o1 > M2) + (o2 > M2);
      ge2 += (o1 >= M2) + (o2 >= M2);
    }
    float mine = -INFINITY;
    if (gt1 < a.k && ge1 >= a.k) mine = M1;
    if (gt2 < a.k && ge2 >= a.k) mine = fmaxf(mine, M2);
    mine = fmaxf(mine, __shfl_xor_sync(FULL, mine, 1));
    mine = fmaxf(mine, __shfl_xor_sync(FULL, mine, 2));
    kth = fmaxf(mine, __shfl_xor_sync(FULL, mine, 4));
  }

  // ---- 4. candidates: listed per token (expert ids), then their exact keys
  //         computed by the token's 8 lanes, entries g, g + 8, ... ----
  const uint32_t cmask = (maybe && tv) ? proxy_mask<NW>(p2, kth - 2.0f * delta) : 0u;
  const int cnt = __popc(cmask);
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    const int o = __shfl_up_sync(FULL, incl, off, 8);
    if (g >= off) incl += o;
  }
  const int total = __shfl_sync(FULL, incl, seg | 7);
  const bool slow = tv && (total > kCandSlots || total < a.k);
  const bool fast = tv && !slow;
  const int pos0 = incl - cnt;
  uint16_t* ce = reinterpret_cast<uint16_t*>(cand + 4 * kCandSlots * 12) + q * kCandSlots;
  if (fast) {
    uint32_t m = cmask;
    for (int pos = pos0; m; ++pos, m &= m - 1) ce[pos] = (uint16_t)slot_expert<V, ESZ>(g, rot, mask_bit_slot(__ffs(m) - 1));
  }
  __syncwarp();
  const int npass = fast ? ((total > 16) ? 2 : 1) : 0;
  for (int ps = 0; ps < npass; ++ps) {
    float kx[2], sx[2];
    int ex[2];
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = g + 8 * (2 * ps + u);
      ok[u] = i < total;
      ex[u] = ok[u] ? ce[i] : 0;
      sx[u] = sigmoid_f32(stage_val(a, row, ex[u]));
      kx[u] = sx[u] + bias_s[ex[u]];
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!ok[u]) continue;
      const int i = g + 8 * (2 * ps + u);
      ck[i] = pack_key(kx[u], ex[u]);
      cs[i] = sx[u];
    }
  }
  if (fast && g == 0 && (total & 1)) ck[total] = 0ull;  // pads the last pair: ranks below every candidate
  __syncwarp();
  // undecided groups: exact scores from their candidates (the lane's own list
  // entries), ranked among themselves for the slots the surely kept groups
  // leave; the dropped ones' candidates rank below every other
  if (__any_sync(FULL, fast && undec)) {
    float X1 = -INFINITY, X2 = -INFINITY;
    if (fast && undec)
      for (int i = pos0; i < pos0 + cnt; ++i) {
        const uint32_t ok32 = (uint32_t)(ck[i] >> 32);  // ordered key -> fp32 key
        const float kx = __uint_as_float((ok32 & 0x80000000u) ? (ok32 & 0x7fffffffu) : ~ok32);
        const float hi = fmaxf(X1, kx);
        X2 = fmaxf(X2, fminf(X1, kx));
        X1 = hi;
      }
    const unsigned sure_b = (__ballot_sync(FULL, maybe && !undec) >> seg) & 0xffu;
    const int free_slots = K - __popc(sure_b);
    const float gx = (a.topn == 1) ? X1 : (X1 + X2);
    int rx = 0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float o = __shfl_sync(FULL, gx, seg | h);
      const bool ou = (__shfl_sync(FULL, undec ? 1 : 0, seg | h) != 0);
      rx += (ou && (o > gx || (o == gx && h < g))) ? 1 : 0;
    }
    __syncwarp();
    if (fast && undec && rx >= free_slots)
      for (int i = pos0; i < pos0 + cnt; ++i) ck[i] = 0ull;
    __syncwarp();
  }

  // ranks: lane g ranks slots g, g + 8, ... against the token's candidates
  const int tot2 = (total + 1) & ~1;
  int rk[4];
  unsigned long long kk[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = g + 8 * r;
    rk[r] = kCandSlots;
    kk[r] = 0ull;
    if (fast && i < total) {
      kk[r] = ck[i];
      rk[r] = kk[r] ? 0 : kCandSlots;
    }
  }
  if (fast) {
    const int nr = (total + 7) >> 3;
    for (int jj = 0; jj < tot2; jj += 2) {
      const ulonglong2 o = *reinterpret_cast<const ulonglong2*>(ck + jj);
      rk[0] += (o.x > kk[0]) + (o.y > kk[0]);
      rk[1] += (o.x > kk[1]) + (o.y > kk[1]);
      if (nr > 2) {
        rk[2] += (o.x > kk[2]) + (o.y > kk[2]);
        rk[3] += (o.x > kk[3]) + (o.y > kk[3]);
      }
    }
  }
  float sel_sum = 0.0f;
#pragma unroll
  for (int r = 0; r < 4; ++r)
    if (rk[r] < a.k) sel_sum += cs[g + 8 * r];
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 1);
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 2);
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 4);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (rk[r] < a.k) {
      const size_t o = (size_t)t * a.kt + rk[r];
      const int e = packed_expert(kk[r]);
      const float sv = cs[g + 8 * r];
      a.ids[o] = e;
      store_from_f32(a.weights, a.weights_dtype, o, a.renorm ? (sv / sel_sum) * a.scale : sv * a.scale);
      mark(a, masks, ids_s, lt, rk[r], e);
    }
  }

  // ---- tokens left to the exact path ----
  const unsigned sb = __ballot_sync(FULL, slow && g == 0);
  return (sb & 1u) | ((sb >> 7) & 2u) | ((sb >> 14) & 4u) | ((sb >> 21) & 8u);
}

// The exact path for one token (warp per token, E / 32 experts per lane), its
// row read from global memory; kept out of line so that its code and registers
// stay away from the fast path.
template <int VPL>
__device__ __noinline__ void select_token_warp_exact(const RouteArgs& a, const uint8_t* lg_bytes, int t_begin,
                                                     int lt, const float* bias_s, uint32_t* masks, uint16_t* ids_s,
                                                     int lane) {
  select_token_warp<VPL>(a, lg_bytes + ((size_t)t_begin + lt) * a.row_bytes, t_begin + lt, lt, bias_s, masks, ids_s,
                         lane);
}

// Exclusive scan of padded counts into offs[0..E] (E <= 1024) by warp 0: lane
// l takes a run of consecutive experts, then one shuffle scan over the lanes.
// Ends with a block barrier.
__device__ void scan_padded_offsets(const int* cnt, int* offs, int E, int tile) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) >> 5;
    const int e0 = lane * per;
    int local = 0;
    const int tm = tile - 1;  // tile is a power of two
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) local += (cnt[e] + tm) & ~tm;
    }
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        offs[e] = run;
        run += (cnt[e] + tm) & ~tm;
      }
    }
    if (lane == 31) offs[E] = incl;
  }
  __syncthreads();
}

// After a block's selections: park (expert, rank in the segment) of every
// selection in expanded_to_permuted, and write the segment's counts row.
__device__ void finish_segment(const RouteArgs& a, const uint32_t* masks, const uint16_t* ids_s, int n, int t_begin) {
  const int n_items = n * a.kt;
  const long long i_begin = (long long)t_begin * a.kt;
  for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
    const int e = ids_s[i];
    // token of item i: i / k (i < 2^13, so the multiply-high is exact)
    const int lt = a.kt == 1 ? i : (int)__umulhi((uint32_t)i, a.kinv);
    const uint32_t* m = masks + min(e, a.E2 - 1) * a.MW;  // ids were range-checked when selected
    int r = __popc(m[lt >> 5] & ((1u << (lt & 31)) - 1u));
    for (int w = 0; w < (lt >> 5); ++w) r += __popc(m[w]);
    a.e2p[i_begin + i] = e < a.E2 ? (e | (r << 16)) : -1;
  }
  uint8_t* trow = a.table + (size_t)blockIdx.x * a.row_stride;
  uint32_t* grow = a.gtot + (size_t)(blockIdx.x / a.GS) * a.E2;
  for (int e = threadIdx.x; e < a.E2; e += blockDim.x) {
    int c = 0;
    for (int w = 0; w < a.MW; ++w) c += __popc(masks[e * a.MW + w]);
    if (a.cnt_bytes == 1) trow[e] = (uint8_t)c;
    else reinterpret_cast<uint16_t*>(trow)[e] = (uint16_t)c;
    if (c) atomicAdd(&grow[e], (uint32_t)c);  // integer adds: order-free, deterministic
  }
}

// bounded wait on a staging barrier; false (recorded) if it gave up
__device__ __forceinline__ bool stage_wait(const RouteArgs& a, uint64_t* bar, uint32_t parity) {
  if (mbar_wait_bounded(bar, parity, a.timeout_ns)) return true;
  record_timeout(a.hdr);
  return false;
}

// VPL: experts per lane (0 = a thread per token).  FAST_ESZ: 0 = generic exact
// path; 2 or 4 = sigmoid fast path with V = VPL and that logits element size.
template <int VPL, int FAST_ESZ>
__global__ void __launch_bounds__((FAST_ESZ > 0) ? kFastWarpsMax * 32 : kGenericThreads, 1)
    route_select_kernel(RouteArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr bool kFast = FAST_ESZ > 0;
  constexpr int FV = kFast ? VPL : 1;
  const int E = a.E;
  const int c = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int t_begin = c * a.B;
  const int n = max(0, min(a.T, t_begin + a.B) - t_begin);
  const SelSmem L = sel_smem_layout(a.E2, a.MW, a.B, a.kt, kFast ? 1 : 0, FV, a.row_bytes, nwarps, a.slots);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + L.masks);
  uint16_t* ids_s = reinterpret_cast<uint16_t*>(smem + L.ids);
  float* bias_s = reinterpret_cast<float*>(smem + L.bias);
  uint8_t* cb_s = smem + L.cb;
  float* delta_s = reinterpret_cast<float*>(smem + L.delta);
  uint8_t* wbase = smem + L.warp0 + (size_t)warp * L.warp_bytes;
  uint8_t* cand = wbase + a.slots * L.stage_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(wbase + a.slots * L.stage_bytes + kCandBytes);

  // Programmatic dependent launch: the bookkeeping kernel may be scheduled at
  // once.  Before waiting on the previous grid, only the bias is read (a
  // preceding kernel that lets its dependents start early must not write it);
  // the logits are read after the wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int i = threadIdx.x; i < a.E2 * a.MW; i += blockDim.x) masks[i] = 0u;
  const int nq = (n + 3) >> 2;
  if constexpr (kFast) {
    if (lane == 0) {
      mbar_init(&bar[0], 1);
      mbar_init(&bar[1], 1);
    }
    __syncwarp();
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    bias_s[e] = a.has_bias ? load_as_f32(a.bias, a.bias_dtype, e) : 0.0f;
  __syncthreads();
  float delta = 0.0f;
  if constexpr (kFast) {
    // per-lane constants 0.5 + bias in f16, in register-slot order; warp 0
    // also derives the block's proxy error bound from their largest magnitude
    for (int idx = threadIdx.x; idx < 8 * FV; idx += blockDim.x) {
      const int g = idx / FV, j = idx % FV;
      const int rot = (g * (FV / (16 / FAST_ESZ))) >> 3;
      reinterpret_cast<__half*>(cb_s + g * cb_stride_bytes<FV>())[j] =
          __float2half_rn(0.5f + bias_s[slot_expert<FV, FAST_ESZ>(g, rot, j)]);
    }
    if (warp == 0) {
      float cbmax = 0.0f;
      for (int e = lane; e < E; e += 32) cbmax = fmaxf(cbmax, fabsf(0.5f + bias_s[e]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cbmax = fmaxf(cbmax, __shfl_xor_sync(0xffffffffu, cbmax, off));
      if (lane == 0) *delta_s = proxy_delta(cbmax, FAST_ESZ == 4);
    }
    __syncthreads();
    delta = *delta_s;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // fast path: this warp's first two quads start streaming into its slots
  const uint8_t* lg_bytes = reinterpret_cast<const uint8_t*>(a.logits);
  if constexpr (kFast) {
    if (lane == 0) {
      for (int s = 0; s < a.slots; ++s) {
        const int qd = warp + s * nwarps;
        if (qd < nq) {
          const uint32_t bytes = (uint32_t)min(4, n - qd * 4) * (uint32_t)a.row_bytes;
          mbar_arrive_expect_tx(&bar[s], bytes);
          bulk_g2s(wbase + s * L.stage_bytes, lg_bytes + ((size_t)t_begin + qd * 4) * a.row_bytes, bytes, &bar[s]);
        }
      }
    }
  }

  if constexpr (kFast) {
    uint16_t* pend = reinterpret_cast<uint16_t*>(cand + kCandBytes - 2 * kPendMax - 8);
    int npend = 0;
    bool ok = true;
    int r = 0;
    for (int qd = warp; qd < nq; qd += nwarps, ++r) {
      const int s = r & 1;
      if (!stage_wait(a, &bar[s], (uint32_t)(r >> 1) & 1u)) {
        ok = false;
        break;
      }
      const uint8_t* slot = wbase + s * L.stage_bytes;
      const unsigned sq = select_quad_fast<FV, FAST_ESZ>(a, slot, qd * 4, min(4, n - qd * 4), t_begin, cb_s, bias_s,
                                                         delta, cand, masks, ids_s, lane);
      // the quad's tokens left to the exact path (rare) wait for the end of the loop
      for (unsigned m = sq; m; m &= m - 1) {
        if (lane == 0 && npend < kPendMax) pend[npend] = (uint16_t)(qd * 4 + __ffs(m) - 1);
        ++npend;
      }
      __syncwarp();
      const int nx = qd + 2 * nwarps;
      if (lane == 0 && nx < nq) {
        // this slot's rows were read through the generic proxy: order those
        // reads before the bulk copy's writes
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const uint32_t bytes = (uint32_t)min(4, n - nx * 4) * (uint32_t)a.row_bytes;
        mbar_arrive_expect_tx(&bar[s], bytes);
        bulk_g2s(wbase + s * L.stage_bytes, lg_bytes + ((size_t)t_begin + nx * 4) * a.row_bytes, bytes, &bar[s]);
      }
    }
    if (!ok) {
      // a staging wait gave up (recorded; outputs undefined): let the copies
      // still in flight (rounds r and r + 1) land before the block exits
      for (int rr = r; rr < r + 2 && warp + rr * nwarps < nq; ++rr)
        mbar_wait_bounded(&bar[rr & 1], (uint32_t)(rr >> 1) & 1u, a.timeout_ns);
    }
    // this warp's tokens left to the exact path
    __syncwarp();
    if (npend > kPendMax && lane == 0) record_bounds(a.hdr);  // cannot happen: see kPendMax
    for (int i = 0; i < min(npend, kPendMax); ++i)
      select_token_warp_exact<FV / 4>(a, lg_bytes, t_begin, pend[i], bias_s, masks, ids_s, lane);
    } else if constexpr (VPL == 0) {
    for (int lt = threadIdx.x; lt < n; lt += blockDim.x) {
      const uint8_t* row = lg_bytes + ((size_t)t_begin + lt) * a.row_bytes;
      if (E <= 8)
        select_token_thread<8>(a, row, t_begin + lt, lt, bias_s, masks, ids_s);
      else if (E <= 16)
        select_token_thread<16>(a, row, t_begin + lt, lt, bias_s, masks, ids_s);
      else
        select_token_thread<32>(a, row, t_begin + lt, lt, bias_s, masks, ids_s);
    }
  } else {
    for (int lt = warp; lt < n; lt += nwarps)
      select_token_warp<VPL>(a, lg_bytes + ((size_t)t_begin + lt) * a.row_bytes, t_begin + lt, lt, bias_s, masks,
                             ids_s, lane);
  }
  // the fused shared experts' slots: every token of the segment, after its k
  // routed slots, expert E + s with weight 1.0 (their masks hold every token)
  if (a.S > 0) {
    for (int i = threadIdx.x; i < n * a.S; i += blockDim.x) {
      const int lt = i / a.S, s = i % a.S;
      const size_t o = ((size_t)t_begin + lt) * a.kt + a.k + s;
      a.ids[o] = E + s;
      store_from_f32(a.weights, a.weights_dtype, o, 1.0f);
      ids_s[lt * a.kt + a.k + s] = (uint16_t)(E + s);
    }
    for (int i = threadIdx.x; i < a.S * a.MW; i += blockDim.x) {
      const int s = i / a.MW, w = i % a.MW;
      const int lo = w * 32, cntw = max(0, min(32, n - lo));
      masks[(E + s) * a.MW + w] = cntw >= 32 ? 0xffffffffu : ((1u << cntw) - 1u);
    }
  }
  __syncthreads();
  finish_segment(a, masks, ids_s, n, t_begin);
}

// ---------------------------------------------------------------------------
// bookkeeping kernel
// ---------------------------------------------------------------------------
__host__ __device__ inline int perm_smem_bytes(int E) { return (3 * E + 1) * 4 + 16; }

__global__ void __launch_bounds__(kPermThreads, 1) route_permute_kernel(RouteArgs a) {
  extern __shared__ __align__(128) uint8_t psmem[];
  const int E = a.E2;  // experts counted: the routed ones, then the fused shared ones
  int* cnt = reinterpret_cast<int*>(psmem);
  int* base = cnt + E;
  int* offs = base + E;  // [E + 1], then one flag word
  const int c = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t_begin = c * a.B;
  const int n = max(0, min(a.T, t_begin + a.B) - t_begin);
  const int n_items = n * a.kt;
  const long long i_begin = (long long)t_begin * a.kt;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the table and the parked ranks are the selection's output

  unsigned int ticket = 0u;  // thread 0: this block's place among those that have read the group totals
  auto release_totals = [&]() {
    __syncthreads();
    if (threadIdx.x == 0) base[E + E + 1] = ticket == (unsigned)a.G - 1 ? 1 : 0;
    __syncthreads();
    if (base[E + E + 1]) {
      for (int i = threadIdx.x; i < a.NG * E; i += kPermThreads) a.gtot[i] = 0u;
      if (threadIdx.x == 0) a.hdr->ticket = 0u;
    }
  };

  // this block's first parked selections, loaded while the table is summed
  constexpr int kPre = 2;
  int pre[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) {
    const int i = threadIdx.x + u * kPermThreads;
    pre[u] = i < n_items ? __ldcg(a.e2p + i_begin + i) : 0;
  }

  // ---- per expert e (a thread each): cnt[e] = all selections of e (local
  //      experts; others zero width) = the sum of the group totals; base[e] =
  //      the selections of e by earlier segments = the groups before this
  //      segment's group plus this group's segments before this one.  Integer
  //      sums in a fixed order, 8 loads in flight. ----
  {
    const int grp = c / a.GS, r0 = grp * a.GS;
    for (int e = threadIdx.x; e < E; e += kPermThreads) {
      uint32_t tot = 0, pre_e = 0;
      // the group totals (at most kMaxGroups) and this group's earlier rows
      // (fewer than GS): the first 16 of each in flight together
      uint32_t vg[kMaxGroups], vr[16];
#pragma unroll
      for (int j = 0; j < kMaxGroups; ++j) vg[j] = j < a.NG ? __ldcg(a.gtot + (size_t)j * E + e) : 0u;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = r0 + j;
        const uint8_t* trow = a.table + (size_t)r * a.row_stride;
        vr[j] = r < c ? (a.cnt_bytes == 1 ? (uint32_t)__ldcg(trow + e)
                                          : (uint32_t)__ldcg(reinterpret_cast<const uint16_t*>(trow) + e))
                      : 0u;
      }
#pragma unroll
      for (int j = 0; j < kMaxGroups; ++j) {
        tot += vg[j];
        pre_e += j < grp ? vg[j] : 0u;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) pre_e += vr[j];
      for (int rb = r0 + 16; rb < c; rb += 8) {  // groups of more than 16 segments (very large T)
        uint32_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = rb + j;
          const uint8_t* trow = a.table + (size_t)r * a.row_stride;
          v[j] = r < c ? (a.cnt_bytes == 1 ? (uint32_t)__ldcg(trow + e)
                                           : (uint32_t)__ldcg(reinterpret_cast<const uint16_t*>(trow) + e))
                       : 0u;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) pre_e += v[j];
      }
      cnt[e] = is_local(a, e) ? (int)tot : 0;  // another shard's expert: zero width
      base[e] = (int)pre_e;
    }
    __syncthreads();
    // this block has read the group totals: take a ticket now, look at it at
    // the end (the last block to have read them clears them for the next call)
    if (threadIdx.x == 0) ticket = atomicAdd(&a.hdr->ticket, 1u);
  }
  scan_padded_offsets(cnt, offs, E, a.tile);
  const int P = offs[E];
  if (c == 0) {
    // the shard's experts, then the shared ones (the others have no rows:
    // offs[loc_off] == 0, and the shared experts follow the shard's)
    for (int le = threadIdx.x; le < a.loc_n + a.S; le += blockDim.x) {
      const int e = le < a.loc_n ? a.loc_off + le : a.E + (le - a.loc_n);
      a.counts[le] = cnt[e];
      a.offsets[le] = offs[e];
    }
    if (threadIdx.x == 0) {
      a.offsets[a.loc_n + a.S] = P;
      a.totals[0] = P;
      a.totals[1] = P / a.tile;
    }
  }

  // ---- slots in token order: offset + earlier segments' rows + rank ----
  for (int i0 = 0; i0 < n_items; i0 += kPre * kPermThreads) {
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int i = i0 + threadIdx.x + u * kPermThreads;
      if (i >= n_items) continue;
      const int v = (i0 == 0) ? pre[u] : __ldcg(a.e2p + i_begin + i);
      const int e = v & 0xffff, rk = v >> 16;
      if (v < 0 || e >= E) {
        record_bounds(a.hdr);
        continue;
      }
      if (!is_local(a, e)) {  // another shard's expert: no slot
        a.e2p[i_begin + i] = -1;
        continue;
      }
      const int slot = offs[e] + base[e] + rk;
      a.e2p[i_begin + i] = slot;
      // token of item i: t_begin + i / k
      const int lt = a.kt == 1 ? i : (int)__umulhi((uint32_t)i, a.kinv);
      if ((unsigned)slot < (unsigned)a.max_padded) a.p2t[slot] = t_begin + lt;
      else record_bounds(a.hdr);
    }
  }

  // ---- tile tables and padding rows: a warp per expert (experts spread over
  //      all warps of the grid); the expert's tiles are [offs[e], offs[e+1]) / tile
  //      and its padding rows follow its count ----
  if (P / a.tile > a.max_tiles || P > a.max_padded) {
    if (threadIdx.x == 0) record_bounds(a.hdr);
    release_totals();
    return;
  }
  const int nwarps = blockDim.x >> 5;
  for (int e = c * nwarps + warp; e < E; e += a.G * nwarps) {
    const int row0 = offs[e], row1 = offs[e + 1], lim = row0 + cnt[e];
    for (int tc = row0 / a.tile + lane; tc < row1 / a.tile; tc += 32) {
      a.tile_expert[tc] = local_index(a, e);  // the local expert (batch index)
      a.tile_mn[tc] = min((tc + 1) * a.tile, lim);
    }
    for (int r = lim + lane; r < row1; r += 32) a.p2t[r] = -1;
  }
  release_totals();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct DevInfo {
  int sms = 0;
  int smem_optin = 0;
};

DevInfo device_info() {
  static DevInfo cache[64];
  static std::once_flag once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::call_once(once[dev], [dev] {
    cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&cache[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  });
  return cache[dev];
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int esize(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

int validate(const moe_route_params* p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  if (p->num_tokens < 0 || p->num_experts <= 0 || p->top_k <= 0 || p->top_k > p->num_experts)
    return MOE_ERR_INVALID_ARG;
  if (p->score_fn != MOE_SOFTMAX && p->score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (p->local_expert_offset < 0 || p->local_num_experts < 0 ||
      (long long)p->local_expert_offset + (p->local_num_experts > 0 ? p->local_num_experts : 1) > p->num_experts ||
      (p->local_num_experts == 0 && p->local_expert_offset != 0))
    return MOE_ERR_INVALID_ARG;
  if ((p->logits_dtype != MOE_F32 && p->logits_dtype != MOE_BF16) ||
      (p->bias_dtype != MOE_F32 && p->bias_dtype != MOE_BF16) ||
      (p->weights_dtype != MOE_F32 && p->weights_dtype != MOE_BF16))
    return MOE_ERR_INVALID_ARG;
  if (!is_pow2(p->tile_tokens_dim) || p->tile_tokens_dim > 4096) return MOE_ERR_INVALID_ARG;
  const bool grouped = p->n_group > 1 && p->topk_group > 0;
  if (grouped) {
    if (p->num_experts % p->n_group != 0) return MOE_ERR_INVALID_ARG;
    const int gs = p->num_experts / p->n_group;
    if (p->group_score_topn < 1 || p->group_score_topn > gs) return MOE_ERR_INVALID_ARG;
    const int kept = std::min(p->topk_group, p->n_group);
    if ((long long)p->top_k > (long long)kept * gs) return MOE_ERR_INVALID_ARG;
    if (p->group_score_topn > 2) return MOE_ERR_UNSUPPORTED;
  }
  if (p->num_fused_shared_experts < 0) return MOE_ERR_INVALID_ARG;
  const int S = p->num_fused_shared_experts;
  if (p->num_experts + S > MOE_MAX_EXPERTS || p->top_k + S > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  const long long items = (long long)p->num_tokens * (p->top_k + S);
  if (items + std::min<long long>(p->num_experts + S, items) * (p->tile_tokens_dim - 1) > 0x7fffffffLL)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

bool group_layout_ok(const moe_route_params* p, int vpl) {
  const bool grouped = p->n_group > 1 && p->topk_group > 0;
  if (!grouped || vpl == 0) return true;
  const int gs = p->num_experts / p->n_group;
  if (gs >= vpl) return (gs % vpl == 0) && is_pow2(gs / vpl) && (gs / vpl) <= 32;
  return (vpl % gs) == 0;
}

// Experts per lane for the warp-per-token path (0 = thread per token): the
// smallest supported width that covers E in one warp and maps every group onto
// whole lanes (or whole groups onto one lane).  -1 if none does.
constexpr int kVplChoices[] = {2, 3, 4, 5, 6, 8, 12, 16, 24, 32};

int pick_mode(const moe_route_params* p) {
  const int E = p->num_experts;
  if (E <= 32) return 0;
  for (int vpl : kVplChoices)
    if (vpl * 32 >= E && group_layout_ok(p, vpl)) return vpl;
  return -1;
}

// Segments: about one per SM (at least 32 tokens each, at most kMaxSegment).
void plan_segments(int T, int sms, int* G, int* B) {
  if (T <= 0) {
    *G = 1;
    *B = 1;
    return;
  }
  const int g = std::max(1, std::min(sms, (T + 31) / 32));
  const int b = std::min(kMaxSegment, (T + g - 1) / g);
  *G = (T + b - 1) / b;
  *B = b;
}

// workspace: header | group totals [16][MOE_MAX_EXPERTS] u32 (at a fixed place
// and size: every call leaves the part it used zero, whatever its shape) |
// table [G][row] (rows of 1- or 2-byte entries, 16-byte multiples)
constexpr size_t kHeaderBytes = 256;
constexpr size_t kTableOffset = kHeaderBytes + (size_t)kMaxGroups * MOE_MAX_EXPERTS * 4;

size_t table_row_stride(int E, int cnt_bytes) { return ((size_t)E * cnt_bytes + 15) & ~(size_t)15; }

size_t ws_bytes_for(int T, int E, int sms) {
  int G = 1, B = 1;
  plan_segments(T, sms, &G, &B);
  return kTableOffset + (size_t)G * table_row_stride(E, B <= 255 ? 1 : 2);
}

// sigmoid fast path: 8 lanes per token, one lane per E/8 experts
bool fast_path_ok(const moe_route_params* p, const void* logits) {
  if (p->score_fn != MOE_SIGMOID || !p->softmax_before_topk) return false;
  if (p->num_experts % 8 != 0 || p->top_k > 8) return false;
  if ((reinterpret_cast<uintptr_t>(logits) & 15) != 0) return false;  // rows staged by bulk copies
  const int V = p->num_experts / 8;
  const bool v_ok = p->logits_dtype == MOE_BF16 ? (V == 8 || V == 16 || V == 32) : (V == 8 || V == 16);
  if (!v_ok) return false;
  const bool grouped = p->n_group > 1 && p->topk_group > 0;
  // the candidate bound needs two experts per kept group to cover k
  if (grouped && (p->n_group != 8 || p->group_score_topn > 2 || 2 * std::min(p->topk_group, 8) < p->top_k))
    return false;
  return true;
}

// Both route kernels ask for the largest shared-memory carveout, so that an
// SM switching from one to the other need not reconfigure its L1 / shared split.
template <typename K>
cudaError_t set_smem_attr(K kernel, int smem) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess || smem <= 48 * 1024) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

template <int VPL, int FAST_ESZ>
cudaError_t launch_select(const RouteArgs& a, int threads, int smem, cudaStream_t st) {
  cudaError_t e = set_smem_attr(route_select_kernel<VPL, FAST_ESZ>, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_select_kernel<VPL, FAST_ESZ>, dim3(a.G), dim3(threads), (size_t)smem, st, a);
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_route_capacity(const moe_route_params* p, int64_t* max_padded, int64_t* max_tiles) {
  const int v = validate(p);
  if (v != MOE_OK) return v;
  if (!max_padded || !max_tiles) return MOE_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)p->num_tokens * (p->top_k + p->num_fused_shared_experts);
  const int64_t nz = std::min<int64_t>(rows, p->num_experts + p->num_fused_shared_experts);
  *max_padded = rows + nz * (p->tile_tokens_dim - 1);
  *max_tiles = *max_padded / p->tile_tokens_dim;
  return MOE_OK;
}

extern "C" int moe_route_workspace_bytes(const moe_route_params* p, size_t* bytes) {
  const int v = validate(p);
  if (v != MOE_OK) return v;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const DevInfo d = device_info();
  if (d.sms <= 0) return MOE_ERR_CUDA;
  *bytes = ws_bytes_for(p->num_tokens, p->num_experts + p->num_fused_shared_experts, d.sms);
  return MOE_OK;
}

extern "C" int moe_route(const moe_route_params* p, const void* logits, const void* bias, int32_t* topk_ids,
                         void* topk_weights, int32_t* expert_counts, int32_t* padded_offsets,
                         int32_t* expanded_to_permuted, int32_t* permuted_to_token, int32_t* tile_expert,
                         int32_t* tile_mn_limit, int32_t* totals, void* ws, size_t ws_bytes, void* stream) {
  const int v = validate(p);
  if (v != MOE_OK) return v;
  const int T = p->num_tokens;
  if ((T > 0 && (!logits || !topk_ids || !topk_weights || !expanded_to_permuted || !permuted_to_token ||
                 !tile_expert || !tile_mn_limit)) ||
      !expert_counts || !padded_offsets || !totals)
    return MOE_ERR_INVALID_ARG;
  const int mode = pick_mode(p);
  if (mode < 0) return MOE_ERR_UNSUPPORTED;
  const DevInfo d = device_info();
  if (d.sms <= 0) return MOE_ERR_CUDA;
  if (!ws || ws_bytes < ws_bytes_for(T, p->num_experts + p->num_fused_shared_experts, d.sms)) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0) return MOE_ERR_WORKSPACE;

  RouteArgs a = {};
  a.logits = logits;
  a.bias = bias;
  a.ids = topk_ids;
  a.weights = topk_weights;
  a.counts = expert_counts;
  a.offsets = padded_offsets;
  a.e2p = expanded_to_permuted;
  a.p2t = permuted_to_token;
  a.tile_expert = tile_expert;
  a.tile_mn = tile_mn_limit;
  a.totals = totals;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  a.table = reinterpret_cast<uint8_t*>(ws) + kTableOffset;
  a.T = T;
  a.E = p->num_experts;
  a.k = p->top_k;
  a.S = p->num_fused_shared_experts;
  a.kt = a.k + a.S;
  a.E2 = a.E + a.S;
  a.score_fn = p->score_fn;
  a.pre = p->softmax_before_topk ? 1 : 0;
  a.grouped = (p->n_group > 1 && p->topk_group > 0) ? 1 : 0;
  a.n_group = p->n_group;
  a.topk_group = std::min(p->topk_group, p->n_group);
  a.topn = p->group_score_topn;
  a.renorm = p->renormalize ? 1 : 0;
  a.scale = p->scaling_factor;
  a.tile = p->tile_tokens_dim;
  a.kinv = a.kt > 1 ? (uint32_t)((0x100000000ull + (uint64_t)a.kt - 1) / (uint64_t)a.kt) : 0u;
  a.logits_dtype = p->logits_dtype;
  a.bias_dtype = p->bias_dtype;
  a.weights_dtype = p->weights_dtype;
  a.has_bias = bias != nullptr;
  plan_segments(T, d.sms, &a.G, &a.B);
  a.MW = (a.B + 31) / 32;
  a.GS = (a.G + kMaxGroups - 1) / kMaxGroups;
  a.NG = (a.G + a.GS - 1) / a.GS;
  a.gtot = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(ws) + kHeaderBytes);
  {
    int64_t mp = 0, mt = 0;
    moe_route_capacity(p, &mp, &mt);
    a.max_padded = (int)mp;
    a.max_tiles = (int)mt;
  }
  a.loc_off = p->local_expert_offset;
  a.loc_n = p->local_num_experts > 0 ? p->local_num_experts : p->num_experts;
  a.row_bytes = p->num_experts * esize(p->logits_dtype);
  a.cnt_bytes = a.B <= 255 ? 1 : 2;
  a.row_stride = (int)table_row_stride(a.E2, a.cnt_bytes);
  a.timeout_ns = kDefaultTimeoutNs;

  const bool fast = fast_path_ok(p, logits);
  int threads;
  if (fast) {
    threads = 32 * std::max(1, std::min(kFastWarpsMax, (a.B + 3) / 4));
  } else if (mode == 0) {
    threads = std::min(kGenericThreads, std::max(32, (a.B + 31) / 32 * 32));
  } else {
    threads = 32 * std::max(1, std::min(kGenericThreads / 32, a.B));
  }
  const int V = a.E / 8;
  a.slots = (fast && (a.B + 3) / 4 > threads / 32) ? 2 : 1;
  const SelSmem L = sel_smem_layout(a.E2, a.MW, a.B, a.kt, fast ? 1 : 0, fast ? V : 1, a.row_bytes, threads / 32,
                                    a.slots);
  if (L.total > d.smem_optin) return MOE_ERR_UNSUPPORTED;
  if ((L.ids | L.bias | L.cb | L.delta | L.warp0) & 15) return MOE_ERR_UNSUPPORTED;  // layout invariant
  const int psmem = perm_smem_bytes(a.E2);
  if (psmem > d.smem_optin) return MOE_ERR_UNSUPPORTED;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (fast) {
    if (p->logits_dtype == MOE_BF16)
      err = V == 8 ? launch_select<8, 2>(a, threads, L.total, st)
          : V == 16 ? launch_select<16, 2>(a, threads, L.total, st)
                    : launch_select<32, 2>(a, threads, L.total, st);
    else
      err = V == 8 ? launch_select<8, 4>(a, threads, L.total, st) : launch_select<16, 4>(a, threads, L.total, st);
  } else {
    switch (mode) {
      case 0: err = launch_select<0, 0>(a, threads, L.total, st); break;
      case 2: err = launch_select<2, 0>(a, threads, L.total, st); break;
      case 3: err = launch_select<3, 0>(a, threads, L.total, st); break;
      case 4: err = launch_select<4, 0>(a, threads, L.total, st); break;
      case 5: err = launch_select<5, 0>(a, threads, L.total, st); break;  // e.g. 160 experts in groups of 20
      case 6: err = launch_select<6, 0>(a, threads, L.total, st); break;
      case 8: err = launch_select<8, 0>(a, threads, L.total, st); break;
      case 12: err = launch_select<12, 0>(a, threads, L.total, st); break;
      case 16: err = launch_select<16, 0>(a, threads, L.total, st); break;
      case 24: err = launch_select<24, 0>(a, threads, L.total, st); break;
      case 32: err = launch_select<32, 0>(a, threads, L.total, st); break;
      default: return MOE_ERR_UNSUPPORTED;
    }
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  err = set_smem_attr(route_permute_kernel, psmem);
  if (err == cudaSuccess)
    err = launch_pdl(route_permute_kernel, dim3(a.G), dim3(kPermThreads), (size_t)psmem, st, a);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// wait test hook: a bounded wait on a barrier that nothing completes
// ---------------------------------------------------------------------------
namespace moe {
namespace {
// One block: thread 0 arms a shared-memory mbarrier for one arrival plus
// `pending` bytes, adds the arrival only when pending == 0, then waits on it
// the way the kernels wait on their bulk copies (bounded).
__global__ void wait_probe_kernel(WsHeader* hdr, uint32_t pending, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_arrive_expect_tx(&bar, pending);  // the arrival; `pending` transaction bytes never come
  if (!mbar_wait_bounded(&bar, 0, timeout_ns)) record_timeout(hdr);
}
}  // namespace
}  // namespace moe

extern "C" int moe_debug_wait_timeout(int32_t never_complete, int64_t timeout_ns, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (timeout_ns <= 0 || timeout_ns > 5LL * 1000 * 1000 * 1000) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<WsHeader*>(ws), never_complete ? 16u : 0u, (long long)timeout_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// proxy error hook
// ---------------------------------------------------------------------------
namespace moe {
namespace {
__global__ void proxy_error_kernel(const float* x, const float* b, long long n, int f32_logits, float* err,
                                   float* delta) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = x[i], cb = 0.5f + b[i];
    const __half2 p = proxy_pair(v, v, __float2half2_rn(cb));
    err[i] = __low2float(p) - (sigmoid_f32(v) + b[i]);
    delta[i] = proxy_delta(fabsf(cb), f32_logits);
  }
}
}  // namespace
}  // namespace moe

extern "C" int moe_debug_sigmoid_proxy_error(const float* x, const float* b, int64_t n, int32_t f32_logits, float* err,
                                             float* delta, void* stream) {
  if (n < 0 || (n > 0 && (!x || !b || !err || !delta))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
  proxy_error_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, b, (long long)n, f32_logits, err,
                                                                               delta);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// moe_route_no_alloc: moe_route with a library-owned, statically allocated
// workspace.
//
// Some callers cannot allocate device memory when they route: code running
// under a memory manager that owns all device memory (a serving runtime that
// reserves the GPU's memory up front and forbids allocations outside its own
// pool), plugin or custom-op interfaces that hand the operator its inputs and
// outputs but no workspace, plain C callers with no device allocator, and
// latency-critical paths that cannot afford cudaMalloc's synchronisation.
// For them the workspace lives in a file-scope __device__ array that every GPU
// loading this library holds until the process exits.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = 512 * 1024;  // the route workspace for E up to a few hundred experts
__device__ __align__(256) uint8_t g_route_scratch[kStaticScratchBytes];

// The array's device address, looked up once per device with that device
// current.  A failed lookup is not cached: the next call tries again.  The
// first successful set-up also zero-fills the array's header and group
// totals on the caller's stream (every call leaves the totals zero again);
// after that the status word is sticky across calls (a recorded error stays
// until moe_route_no_alloc_status clears it).
struct ScratchSlot {
  std::mutex m;
  std::atomic<void*> ptr{nullptr};
};
ScratchSlot g_scratch_slot[64];

void* scratch_address(int dev, cudaStream_t st) {
  ScratchSlot& slot = g_scratch_slot[dev];
  void* p = slot.ptr.load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(slot.m);
  p = slot.ptr.load(std::memory_order_relaxed);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return nullptr;
  }
  if (cudaMemsetAsync(p, 0, kTableOffset, st) != cudaSuccess) return nullptr;  // header and group totals
  slot.ptr.store(p, std::memory_order_release);
  return p;
}

int current_device(int* dev) {
  return (cudaGetDevice(dev) == cudaSuccess && *dev >= 0 && *dev < 64) ? MOE_OK : MOE_ERR_CUDA;
}

__global__ void no_alloc_record_kernel(int32_t code) {
  atomicCAS(&reinterpret_cast<WsHeader*>(g_route_scratch)->status, MOE_OK, code);
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_no_alloc(const moe_route_params* p, const void* logits, const void* bias,
                                  int32_t* topk_ids, void* topk_weights, int32_t* expert_counts,
                                  int32_t* padded_offsets, int32_t* expanded_to_permuted,
                                  int32_t* permuted_to_token, int32_t* tile_expert, int32_t* tile_mn_limit,
                                  int32_t* totals, void* stream) {
  const int v = validate(p);
  if (v != MOE_OK) return v;
  const DevInfo d = device_info();
  if (d.sms <= 0) return MOE_ERR_CUDA;
  if (ws_bytes_for(p->num_tokens, p->num_experts + p->num_fused_shared_experts, d.sms) > kStaticScratchBytes)
    return MOE_ERR_WORKSPACE;
  int dev = 0;
  if (current_device(&dev) != MOE_OK) return MOE_ERR_CUDA;
  void* ws = scratch_address(dev, reinterpret_cast<cudaStream_t>(stream));
  if (!ws) return MOE_ERR_CUDA;
  return moe_route(p, logits, bias, topk_ids, topk_weights, expert_counts, padded_offsets, expanded_to_permuted,
                   permuted_to_token, tile_expert, tile_mn_limit, totals, ws, kStaticScratchBytes, stream);
}

extern "C" int moe_route_no_alloc_status(void* stream, int32_t* status, int clear) {
  if (!status) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (current_device(&dev) != MOE_OK) return MOE_ERR_CUDA;
  void* ws = scratch_address(dev, reinterpret_cast<cudaStream_t>(stream));
  if (!ws) return MOE_ERR_CUDA;
  return moe_status(ws, stream, status, clear);
}

extern "C" int moe_debug_no_alloc_record(int32_t code, void* stream) {
  if (code >= 0) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (current_device(&dev) != MOE_OK) return MOE_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!scratch_address(dev, st)) return MOE_ERR_CUDA;
  no_alloc_record_kernel<<<1, 1, 0, st>>>(code);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
