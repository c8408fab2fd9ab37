// moe_route: expert selection, routing weights and permutation bookkeeping in
// one cooperative launch.
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
// Kernel structure (one block per SM, all blocks co-resident):
//   phase 1  each block owns a contiguous token range; its logits arrive in
//            shared memory by up to 8 1-D bulk copies (TMA), each with its own
//            mbarrier, all issued up front so compute starts on the first one
//            while the rest stream in; each token is scored and selected, its
//            ids/weights written, and a block histogram of expert counts kept
//            in shared memory.  Selection paths:
//              - sigmoid fast path (E = 8*V): 8 lanes per token, a lane per
//                V experts (one expert group when n_group = 8), 4 tokens per
//                warp.  A proxy key from tanh.approx (error <= delta) bounds
//                where the exact keys can matter: exact fp32 keys (the stated
//                formula) are computed only for each lane's top-2 region (exact
//                group scores) and for the candidate set of the top-k, which is
//                then ranked by counting.  Tokens whose candidate set overflows
//                fall back to exact keys for all their experts (slow path);
//              - generic: a warp per token (E > 32) or a thread per token
//                (E <= 32) with exact keys and k rounds of argmax;
//   publish  the block's histogram row goes to the workspace table and is
//            added to the global counts (integer atomics, order-free);
//   barrier  one bounded grid barrier;
//   phase 2  every block derives the padded offsets from the counts, its own
//            base per expert from the earlier blocks' rows, then walks its
//            selections in token order (warp match + popcount) to assign slots
//            deterministically; it also writes its share of the tile tables
//            and of the padding rows of permuted_to_token.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace moe {

namespace {

// threads per block: the sigmoid fast path keeps few registers and runs 24
// warps per SM; the generic paths keep larger per-thread arrays and run 16
constexpr int kThreadsFast = 896;
constexpr int kThreadsGeneric = 512;
constexpr int kWarpsMax = kThreadsFast / 32;
constexpr int kStageBytesMax = 96 * 1024;
constexpr int kMaxSub = 8;         // bulk copies (and mbarriers) per staged round
constexpr int kCandMax = 32;       // fast path: candidate slots per token
constexpr int kCandStride = 33;    // padded so the 4 tokens of a warp hit different banks
// |proxy key - exact key| bound used by the fast path.  The proxy is
// 0.5*tanh.approx(x/2) + (0.5 + b); tanh.approx.f32 has a relative error of
// about 2^-11, i.e. <= 2^-12 on the sigmoid; 2^-10 leaves a 4x margin (the
// margin is checked exhaustively over all bf16 inputs by the test suite).
constexpr float kProxyDelta = 1.0f / 1024.0f;

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
  uint32_t* table;   // [G][row_stride bytes]: per-block expert counts
  int T, E, k;
  int score_fn, pre, grouped, n_group, topk_group, topn;
  int renorm;
  float scale;
  int tile;          // power of two
  uint32_t kinv;     // ceil(2^32 / k): item -> token by a multiply-high
  int logits_dtype, bias_dtype, weights_dtype;
  int has_bias;
  int G;
  int max_padded;
  int max_tiles;
  int loc_off, loc_n;  // the local experts [loc_off, loc_off + loc_n): only they get slots and tiles
  int chunk_tokens;
  int stage_bytes;  // stage region: >= chunk_tokens * row_bytes and >= phase 2's partials
  int row_bytes;
  int cnt_bytes;   // width of a block's histogram entry in the table: 1, 2 or 4
  int row_stride;  // bytes per table row (16-byte multiple)
  int fast;        // 1: sigmoid fast path
  int ids_in_smem; // 1: the block's selections also kept in shared memory (u16)
  long long timeout_ns;
};

struct RouteSmem {
  // offsets (bytes) inside dynamic shared memory
  int stage, cand, bias, hist_cta, hist_w, offs, cnt, bar, flag, scan, ids, lrank, lut, total;
};

// per warp: 4 tokens x kCandStride packed u64 keys, then 4 x kCandStride fp32 scores
__host__ __device__ inline int cand_bytes_per_warp() { return 4 * kCandStride * 12; }

__host__ __device__ inline RouteSmem route_smem_layout(int E, int stage_bytes, int ids_bytes, int nwarps,
                                                       int lut_bytes) {
  RouteSmem L;
  int o = 0;
  L.stage = o;
  o += (stage_bytes + 127) & ~127;
  L.cand = o;
  o += nwarps * cand_bytes_per_warp() + 8 * (32 + 4) * 4;  // + the fast path's per-lane bias table
  L.bias = o;
  o += ((E * 4) + 15) & ~15;
  L.hist_cta = o;
  o += ((E * 4) + 15) & ~15;
  L.hist_w = o;
  o += ((nwarps * E * 4) + 15) & ~15;
  L.offs = o;
  o += (((E + 1) * 4) + 15) & ~15;
  L.cnt = o;
  o += ((E * 4) + 15) & ~15;
  L.bar = o;
  o += 8 * kMaxSub;
  L.flag = o;
  o += 16;
  L.scan = o;
  o += 32 * 4;
  L.ids = o;
  o += (ids_bytes + 15) & ~15;
  L.lrank = o;  // per selection: rank among the block's selections of the same expert (u16)
  o += (ids_bytes + 15) & ~15;
  L.lut = o;
  o += (lut_bytes + 15) & ~15;
  L.total = o;
  return L;
}

// -------------------------------------------------------------------------
// staging: tokens [t0, t0+n) of logits into shared memory
// -------------------------------------------------------------------------
// Issues up to kMaxSub bulk copies, sub-copy s completing on bar[s].  Returns
// their number; 0 means the rows were copied with plain loads instead
// (unaligned source or rows that are not 16-byte multiples) and are ready.
__device__ int stage_issue(const RouteArgs& a, uint8_t* stage, uint64_t* bar, int t0, int n) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(a.logits) + (size_t)t0 * a.row_bytes;
  const bool bulk = ((reinterpret_cast<uintptr_t>(src) & 15) == 0) && (a.row_bytes % 16 == 0);
  if (!bulk) {
    const uint32_t bytes = (uint32_t)n * (uint32_t)a.row_bytes;
    for (uint32_t i = threadIdx.x; i < bytes; i += blockDim.x) stage[i] = src[i];
    __syncthreads();
    return 0;
  }
  const int nsub = min(kMaxSub, n);
  if (threadIdx.x == 0) {
    // earlier generic-proxy accesses of the stage precede the async-proxy writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // every mbarrier completes exactly one phase per round (unused ones with
    // zero bytes), so the parity of round r is r & 1 for all of them
    for (int s = 0; s < kMaxSub; ++s) {
      if (s < nsub) {
        const int tb = s * n / nsub, te = (s + 1) * n / nsub;
        const uint32_t bytes = (uint32_t)(te - tb) * (uint32_t)a.row_bytes;
        mbar_arrive_expect_tx(&bar[s], bytes);
        bulk_g2s(stage + (size_t)tb * a.row_bytes, src + (size_t)tb * a.row_bytes, bytes, &bar[s]);
      } else {
        mbar_arrive_expect_tx(&bar[s], 0u);
      }
    }
  }
  return nsub;
}

// sub-copy holding local token lt when n tokens are split into nsub parts
__device__ __forceinline__ int sub_of(int lt, int n, int nsub) { return ((lt + 1) * nsub - 1) / n; }

__device__ __forceinline__ bool stage_wait(const RouteArgs& a, uint64_t* bar, int s, uint32_t parity) {
  if (mbar_wait_bounded(&bar[s], parity, a.timeout_ns)) return true;
  record_timeout(a.hdr);
  return false;
}

__device__ __forceinline__ float stage_val(const RouteArgs& a, const uint8_t* row, int e) {
  if (a.logits_dtype == MOE_BF16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(row)[e]);
  return reinterpret_cast<const float*>(row)[e];
}

__device__ __forceinline__ float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

// Exact sigmoid of a bf16 input by table: the kernel fills the table with the
// very expression above for every bf16 value with biased exponent in
// [kLutExpLo, kLutExpHi], both signs (8448 entries, 33 KB), so a lookup returns
// exactly what sigmoid_f32 returns.  Inputs outside the range (|x| < 2^-25 or
// |x| >= 2^8, and non-finite) are evaluated directly.
constexpr int kLutExpLo = 102, kLutExpHi = 134;
constexpr int kLutPerSign = (kLutExpHi - kLutExpLo + 1) * 128;
constexpr int kLutEntries = 2 * kLutPerSign;

__device__ __forceinline__ int lut_index(uint32_t b16) {
  const int ex = (int)((b16 >> 7) & 0xffu);
  if (ex < kLutExpLo || ex > kLutExpHi) return -1;
  return (int)(b16 >> 15) * kLutPerSign + (ex - kLutExpLo) * 128 + (int)(b16 & 0x7fu);
}

__device__ __forceinline__ uint32_t lut_bits(int idx) {
  const int sgn = idx / kLutPerSign, r = idx % kLutPerSign;
  return ((uint32_t)sgn << 15) | ((uint32_t)(r / 128 + kLutExpLo) << 7) | (uint32_t)(r % 128);
}

// exact score of expert e of a staged bf16 row: table when available
__device__ __forceinline__ float sigmoid_bf16_row(const float* lut, const uint8_t* row, int e) {
  const uint32_t b16 = reinterpret_cast<const uint16_t*>(row)[e];
  const int idx = lut ? lut_index(b16) : -1;
  return idx >= 0 ? lut[idx] : sigmoid_f32(bf16_bits_to_f32((uint16_t)b16));
}

// -------------------------------------------------------------------------
// warp per token (E > 32): lane l owns experts [l*VPL, l*VPL + VPL)
// -------------------------------------------------------------------------
// keep a copy of a selection in the block's shared-memory id list (phase 2
// reads it instead of global memory)
// expert e belongs to this shard: it gets rows, slots and tiles (phase 1
// counts every expert; phase 2 gives the others zero width)
__device__ __forceinline__ bool is_local(const RouteArgs& a, int e) {
  return (unsigned)(e - a.loc_off) < (unsigned)a.loc_n;
}

__device__ __forceinline__ void keep_id(uint16_t* ids_s, int local_item, int e) {
  if (ids_s) ids_s[local_item] = (uint16_t)e;
}

template <int VPL>
__device__ void select_token_warp(const RouteArgs& a, const uint8_t* row, int t, const float* bias_s,
                                  int* hist_cta, int lane, uint16_t* ids_s, int t_base) {
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
    const size_t o = (size_t)t * a.k + lane;
    a.ids[o] = my_id;
    keep_id(ids_s, (t - t_base) * a.k + lane, my_id);
    store_from_f32(a.weights, a.weights_dtype, o, v);
    if ((unsigned)my_id < (unsigned)E) atomicAdd(&hist_cta[my_id], 1); else record_bounds(a.hdr);
  }
}

// -------------------------------------------------------------------------
// thread per token (E <= EMAX <= 32)
// -------------------------------------------------------------------------
template <int EMAX>
__device__ void select_token_thread(const RouteArgs& a, const uint8_t* row, int t, const float* bias_s,
                                    int* hist_cta, uint16_t* ids_s, int t_base) {
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
      const size_t o = (size_t)t * a.k + j;
      a.ids[o] = sel[j];
      keep_id(ids_s, (t - t_base) * a.k + j, sel[j]);
      store_from_f32(a.weights, a.weights_dtype, o, w);
      if ((unsigned)sel[j] < (unsigned)E) atomicAdd(&hist_cta[sel[j]], 1); else record_bounds(a.hdr);
    }
  }
}

// -------------------------------------------------------------------------
// sigmoid fast path: 8 lanes per token, lane g owns experts [g*V, (g+1)*V)
// -------------------------------------------------------------------------
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Per-lane constants 0.5 + bias of the lane's experts, in register-slot order,
// one padded row of V + 4 floats per lane position g: the 16-byte loads of the
// 8 lanes of a token fall in distinct bank groups.
template <int V>
__host__ __device__ constexpr int cb_stride() { return V + 4; }

// Out-of-line exact selection of one token (rare): exact keys for all experts
// of the lane, exact group scores, k rounds of segment argmax.
template <int V, int ESZ>
__device__ __noinline__ void select_token_exact8(const RouteArgs& a, const uint8_t* row, long long t, int g, int rot,
                                                 int seg, unsigned smask, const float* bias_s, int* hist_cta,
                                                 uint16_t* ids_s, int t_base) {
  constexpr uint32_t VMASK = (V >= 32) ? 0xffffffffu : ((1u << V) - 1u);
  float p[V];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int e = slot_expert<V, ESZ>(g, rot, j);
    p[j] = sigmoid_f32(stage_val(a, row, e)) + bias_s[e];
  }
  uint32_t allowed = VMASK;
  if (a.grouped) {
    float e1 = -INFINITY, e2 = -INFINITY;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float hi = fmaxf(e1, p[j]);
      e2 = fmaxf(e2, fminf(e1, p[j]));
      e1 = hi;
    }
    const float gsc = (a.topn == 1) ? e1 : (e1 + e2);
    int rank = 0;
    for (int h = 0; h < 8; ++h) {
      const float o = __shfl_sync(smask, gsc, seg | h);
      rank += (o > gsc || (o == gsc && h < g)) ? 1 : 0;
    }
    if (rank >= a.topk_group) allowed = 0;
  }
  float ssum = 0.0f;
  for (int jr = 0; jr < a.k; ++jr) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if ((allowed >> j) & 1u) {
        const unsigned long long pk = pack_key(p[j], slot_expert<V, ESZ>(g, rot, j));
        best = pk > best ? pk : best;
      }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      const unsigned long long o = shfl_xor_u64(smask, best, off);
      best = o > best ? o : best;
    }
    const int win = packed_expert(best);
    if (win / V == g) allowed &= ~(1u << expert_slot<V, ESZ>(g, rot, win));
    if (g == 0) {
      const float sg = sigmoid_f32(stage_val(a, row, win));
      a.ids[(size_t)t * a.k + jr] = win;
      keep_id(ids_s, (int)(t - t_base) * a.k + jr, win);
      ssum = ssum + sg;
      if ((unsigned)win < (unsigned)a.E) atomicAdd(&hist_cta[win], 1); else record_bounds(a.hdr);
    }
  }
  if (g == 0) {
    for (int jr = 0; jr < a.k; ++jr) {
      const size_t o = (size_t)t * a.k + jr;
      const float sg = sigmoid_f32(stage_val(a, row, a.ids[o]));
      store_from_f32(a.weights, a.weights_dtype, o, a.renorm ? (sg / ssum) * a.scale : sg * a.scale);
    }
  }
}

template <int V, int ESZ>
__device__ void select_quad_fast(const RouteArgs& a, const uint8_t* stage, int lt_base, int n, int t_round0,
                                 const float* cb_s, const float* bias_s, float* cand, int* hist_cta,
                                 int lane, uint16_t* ids_s, int t_base, const float* lut) {
  constexpr int EPC = 16 / ESZ, NC = V / EPC;
  constexpr uint32_t VMASK = (V >= 32) ? 0xffffffffu : ((1u << V) - 1u);
  const unsigned FULL = 0xffffffffu;
  const int q = lane >> 3, g = lane & 7, seg = lane & 24;
  const int rot = (g * NC) >> 3;
  const int lt = lt_base + q;
  const bool tv = lt < n;
  const uint8_t* row = stage + (size_t)(tv ? lt : 0) * a.row_bytes;
  const long long t = (long long)t_round0 + lt;

  // ---- proxy keys (|p - key| <= kProxyDelta) and their top-2 ----
  float p[V];
  float m1 = -INFINITY, m2 = -INFINITY, n1 = -INFINITY, n2 = -INFINITY;
  const float* cbl = cb_s + g * cb_stride<V>();
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int cc = (c + rot) & (NC - 1);
    const uint4 v = *reinterpret_cast<const uint4*>(row + (size_t)g * V * ESZ + cc * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float cbv[EPC];
#pragma unroll
    for (int i = 0; i < EPC; i += 4) {
      const float4 b4 = *reinterpret_cast<const float4*>(cbl + c * EPC + i);
      cbv[i] = b4.x; cbv[i + 1] = b4.y; cbv[i + 2] = b4.z; cbv[i + 3] = b4.w;
    }
#pragma unroll
    for (int i = 0; i < EPC; ++i) {
      float x;
      if constexpr (ESZ == 2)
        x = __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
      else
        x = __uint_as_float(w[i]);
      const int j = c * EPC + i;
      const float pj = fmaf(0.5f, tanh_approx(0.5f * x), cbv[i]);
      p[j] = pj;
      // two independent top-2 trackers (even / odd slots) shorten the dependency chain
      if ((i & 1) == 0) {
        const float hi = fmaxf(m1, pj);
        m2 = fmaxf(m2, fminf(m1, pj));
        m1 = hi;
      } else {
        const float hi = fmaxf(n1, pj);
        n2 = fmaxf(n2, fminf(n1, pj));
        n1 = hi;
      }
    }
  }
  {
    const float hi = fmaxf(m1, n1);
    m2 = fmaxf(fminf(m1, n1), fmaxf(m2, n2));
    m1 = hi;
  }

  // ---- exact top-2 keys of the lane: evaluated where the proxy is within
  //      2*delta of the lane's 2nd-best proxy (the exact top-2 lie there) ----
  float K1 = -INFINITY, K2 = -INFINITY, S1 = 0.0f, S2 = 0.0f;
  int j1 = -1, j2 = -1;
  if (tv) {
    const float th = m2 - 2.0f * kProxyDelta;
    uint32_t mq[4] = {0u, 0u, 0u, 0u};  // independent partial masks
#pragma unroll
    for (int j = 0; j < V; ++j) mq[j & 3] |= (p[j] >= th ? 1u : 0u) << j;
    uint32_t m = (mq[0] | mq[1]) | (mq[2] | mq[3]);
    while (m) {
      // up to 4 members per pass, their exact keys evaluated side by side
      int jb[4];
      float kb4[4], sb4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        jb[u] = m ? __ffs(m) - 1 : -1;
        m &= m - 1;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = slot_expert<V, ESZ>(g, rot, max(jb[u], 0));
        sb4[u] = (ESZ == 2) ? sigmoid_bf16_row(lut, row, e) : sigmoid_f32(stage_val(a, row, e));
        kb4[u] = sb4[u] + bias_s[e];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (jb[u] < 0) continue;
        const float K = kb4[u];
        if (K > K1) {
          K2 = K1; S2 = S1; j2 = j1;
          K1 = K; S1 = sb4[u]; j1 = jb[u];
        } else if (K > K2) {
          K2 = K; S2 = sb4[u]; j2 = jb[u];
        }
      }
    }
  }

  // ---- kept groups from exact group scores (lane g = group g) ----
  bool kept = true;
  unsigned kb = 0xffu;
  if (a.grouped) {
    const float gsc = (a.topn == 1) ? K1 : (K1 + K2);
    int rank = 0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float o = __shfl_sync(FULL, gsc, seg | h);
      rank += (o > gsc || (o == gsc && h < g)) ? 1 : 0;
    }
    kept = rank < a.topk_group;
    kb = (__ballot_sync(FULL, kept) >> seg) & 0xffu;
  }

  // ---- candidates: every kept lane holds two exact keys >= K2min, so the
  //      k-th largest key is >= K2min when 2 * nkept >= k; any expert that can
  //      reach the top-k has key >= K2min, hence proxy >= K2min - delta ----
  float k2min = kept ? K2 : INFINITY;
  k2min = fminf(k2min, __shfl_xor_sync(FULL, k2min, 1));
  k2min = fminf(k2min, __shfl_xor_sync(FULL, k2min, 2));
  k2min = fminf(k2min, __shfl_xor_sync(FULL, k2min, 4));
  const int nkept = __popc(kb);
  const float tau = (2 * nkept >= a.k) ? (k2min - kProxyDelta) : -INFINITY;
  uint32_t mask = 0;
  if (kept && tv) {
    uint32_t mq[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < V; ++j) mq[j & 3] |= (p[j] >= tau ? 1u : 0u) << j;
    mask = (mq[0] | mq[1]) | (mq[2] | mq[3]);
    if (j1 >= 0) mask |= 1u << j1;
    if (j2 >= 0) mask |= 1u << j2;
  }
  const int cnt = __popc(mask);
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    const int o = __shfl_up_sync(FULL, incl, off, 8);
    if (g >= off) incl += o;
  }
  const int total = __shfl_sync(FULL, incl, seg | 7);
  const bool slow = tv && (total > kCandMax);

  // ---- fast: exact keys of the candidates, ranked by counting on packed
  //      (ordered key, ~expert) words: larger key first, then lower expert ----
  unsigned long long* ck = reinterpret_cast<unsigned long long*>(cand) + q * kCandStride;
  float* cs = cand + 8 * kCandStride + q * kCandStride;
  if (tv && !slow) {
    int pos = incl - cnt;
    uint32_t m = mask;
    if (j1 >= 0) m &= ~(1u << j1);
    if (j2 >= 0) m &= ~(1u << j2);
    // the lane's top-2 (exact already), then the other candidates 4 per pass
    if (j1 >= 0 && ((mask >> j1) & 1u)) {
      ck[pos] = pack_key(K1, slot_expert<V, ESZ>(g, rot, j1));
      cs[pos++] = S1;
    }
    if (j2 >= 0 && ((mask >> j2) & 1u)) {
      ck[pos] = pack_key(K2, slot_expert<V, ESZ>(g, rot, j2));
      cs[pos++] = S2;
    }
    while (m) {
      int jb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        jb[u] = m ? __ffs(m) - 1 : -1;
        m &= m - 1;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = slot_expert<V, ESZ>(g, rot, max(jb[u], 0));
        const float sg = (ESZ == 2) ? sigmoid_bf16_row(lut, row, e) : sigmoid_f32(stage_val(a, row, e));
        if (jb[u] >= 0) {
          ck[pos] = pack_key(sg + bias_s[e], e);
          cs[pos++] = sg;
        }
      }
    }
  }
  __syncwarp();
  constexpr int RPL = kCandMax / 8;  // candidates ranked per lane
  int my_rank[RPL], my_e[RPL];
  float my_s[RPL];
  float sel_sum = 0.0f;
#pragma unroll
  for (int r = 0; r < RPL; ++r) {
    my_rank[r] = kCandMax;
    my_e[r] = 0;
    my_s[r] = 0.0f;
    const int i = g + 8 * r;
    if (tv && !slow && i < total) {
      const unsigned long long ki = ck[i];
      int rank = 0;
      for (int jj = 0; jj < total; ++jj) rank += (ck[jj] > ki) ? 1 : 0;
      my_rank[r] = rank;
      my_e[r] = packed_expert(ki);
      my_s[r] = cs[i];
      if (rank < a.k) sel_sum += my_s[r];
    }
  }
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 1);
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 2);
  sel_sum += __shfl_xor_sync(FULL, sel_sum, 4);
  if (tv && !slow) {
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
      if (my_rank[r] < a.k) {
        const size_t o = (size_t)t * a.k + my_rank[r];
        const float wv = a.renorm ? (my_s[r] / sel_sum) * a.scale : my_s[r] * a.scale;
        a.ids[o] = my_e[r];
        keep_id(ids_s, (int)(t - t_base) * a.k + my_rank[r], my_e[r]);
        store_from_f32(a.weights, a.weights_dtype, o, wv);
        atomicAdd(&hist_cta[my_e[r]], 1);
      }
    }
  }
  __syncwarp();

  // ---- slow: exact keys for every expert of the token (rare) ----
  const unsigned smask = __ballot_sync(FULL, slow);
  if (slow) select_token_exact8<V, ESZ>(a, row, t, g, rot, seg, smask, bias_s, hist_cta, ids_s, t_base);
  __syncwarp();
}

// Exclusive scan of padded counts into offs[0..E] (E <= 1024) by warp 0: lane
// l takes a run of consecutive experts, then one shuffle scan over the lanes.
// Ends with a block barrier.
__device__ void scan_padded_offsets(const int* cnt, int* offs, int E, int tile, int* /*scratch*/) {
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

// VPL: experts per lane (0 = a thread per token).  FAST_ESZ: 0 = generic exact
// path; 2 or 4 = sigmoid fast path with V = VPL and that logits element size.
template <int VPL, int FAST_ESZ>
__global__ void __launch_bounds__((FAST_ESZ > 0) ? kThreadsFast : kThreadsGeneric, 1) route_kernel(RouteArgs a) {
  constexpr int kWarps = ((FAST_ESZ > 0) ? kThreadsFast : kThreadsGeneric) / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  const int E = a.E;
  const int c = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // contiguous token range of this block
  const int base_n = a.T / a.G, rem = a.T % a.G;
  const int t_begin = c * base_n + min(c, rem);
  const int t_end = t_begin + base_n + (c < rem ? 1 : 0);
  const int n_items = (t_end - t_begin) * a.k;
  const RouteSmem L = route_smem_layout(E, a.stage_bytes, a.ids_in_smem ? n_items * 2 : 0, kWarps,
                                       FAST_ESZ == 2 ? kLutEntries * 4 : 0);
  uint8_t* stage = smem + L.stage;
  float* bias_s = reinterpret_cast<float*>(smem + L.bias);
  int* hist_cta = reinterpret_cast<int*>(smem + L.hist_cta);
  int* hist_w = reinterpret_cast<int*>(smem + L.hist_w);
  int* offs = reinterpret_cast<int*>(smem + L.offs);
  int* cnt = reinterpret_cast<int*>(smem + L.cnt);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.bar);
  int* flag = reinterpret_cast<int*>(smem + L.flag);
  int* scan_scratch = reinterpret_cast<int*>(smem + L.scan);
  uint16_t* ids_s = a.ids_in_smem ? reinterpret_cast<uint16_t*>(smem + L.ids) : nullptr;
  uint16_t* lrank_s = a.ids_in_smem ? reinterpret_cast<uint16_t*>(smem + L.lrank) : nullptr;

  // Programmatic dependent launch: the next grid in the stream may be scheduled
  // at once (its blocks start as this grid's blocks retire), and this grid
  // touches no global memory before the previous one has completed and its
  // writes are visible.  Without the launch attribute both are no-ops.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // bf16 fast path: the exact-sigmoid table needs no global memory, so all
  // threads but thread 0 (which waits first and starts the logits copies)
  // fill it before waiting
  float* lut = nullptr;
  if constexpr (FAST_ESZ == 2) {
    lut = reinterpret_cast<float*>(smem + L.lut);
    if (threadIdx.x > 0)
      for (int i = threadIdx.x - 1; i < kLutEntries; i += blockDim.x - 1)
        lut[i] = sigmoid_f32(bf16_bits_to_f32((uint16_t)lut_bits(i)));
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const uint32_t gen = barrier_generation(a.hdr);

  // the first round's logits start streaming before anything else: thread 0
  // initialises the mbarriers and issues the bulk copies itself
  const int n0 = min(a.chunk_tokens, t_end - t_begin);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxSub; ++s) mbar_init(&bar[s], 1);
    flag[1] = 0;  // set when a staging wait gave up
  }
  int nsub = (n0 > 0) ? stage_issue(a, stage, bar, t_begin, n0) : 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    bias_s[e] = a.has_bias ? load_as_f32(a.bias, a.bias_dtype, e) : 0.0f;
    hist_cta[e] = 0;
  }
  __syncthreads();

  // fast path: per-lane constants 0.5 + bias, in register-slot order
  constexpr int FV = (FAST_ESZ > 0) ? VPL : 1;
  float* cb_s = reinterpret_cast<float*>(smem + L.cand + kWarps * cand_bytes_per_warp());
  if constexpr (FAST_ESZ > 0) {
    for (int idx = threadIdx.x; idx < 8 * FV; idx += blockDim.x) {
      const int g = idx / FV, j = idx % FV;
      const int rot = (g * (FV / (16 / FAST_ESZ))) >> 3;
      cb_s[g * cb_stride<FV>() + j] = 0.5f + bias_s[slot_expert<FV, FAST_ESZ>(g, rot, j)];
    }
    __syncthreads();
  }
  float* cand = reinterpret_cast<float*>(smem + L.cand + warp * cand_bytes_per_warp());

  // ---------------- phase 1: select ----------------
  uint32_t round = 0;
  for (int t0 = t_begin; t0 < t_end; t0 += a.chunk_tokens, ++round) {
    const int n = min(a.chunk_tokens, t_end - t0);
    if (round > 0) nsub = stage_issue(a, stage, bar, t0, n);
    const uint32_t parity = round & 1u;
    if constexpr (FAST_ESZ > 0) {
      const int nquads = (n + 3) >> 2;
      for (int qd = warp; qd < nquads; qd += kWarps) {
        if (nsub > 0) {
          const int s0 = sub_of(qd * 4, n, nsub), s1 = sub_of(min(qd * 4 + 3, n - 1), n, nsub);
          for (int sb = s0; sb <= s1; ++sb)
            if (!stage_wait(a, bar, sb, parity)) flag[1] = 1;
        }
        select_quad_fast<FV, FAST_ESZ>(a, stage, qd * 4, n, t0, cb_s, bias_s, cand, hist_cta, lane, ids_s, t_begin,
                                       lut);
      }
    } else {
      for (int sb = 0; sb < nsub; ++sb)
        if (!stage_wait(a, bar, sb, parity)) flag[1] = 1;
      if constexpr (VPL == 0) {
        for (int lt = threadIdx.x; lt < n; lt += blockDim.x) {
          const uint8_t* row = stage + (size_t)lt * a.row_bytes;
          if (E <= 8)
            select_token_thread<8>(a, row, t0 + lt, bias_s, hist_cta, ids_s, t_begin);
          else if (E <= 16)
            select_token_thread<16>(a, row, t0 + lt, bias_s, hist_cta, ids_s, t_begin);
          else
            select_token_thread<32>(a, row, t0 + lt, bias_s, hist_cta, ids_s, t_begin);
        }
      } else {
        for (int lt = warp; lt < n; lt += kWarps)
          select_token_warp<VPL>(a, stage + (size_t)lt * a.row_bytes, t0 + lt, bias_s, hist_cta, lane, ids_s,
                                 t_begin);
      }
    }
    __syncthreads();
  }
  const bool staged_ok = flag[1] == 0;

  // ---------------- publish + barrier ----------------
  uint8_t* trow = reinterpret_cast<uint8_t*>(a.table) + (size_t)c * a.row_stride;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int h = hist_cta[e];
    if (a.cnt_bytes == 1) trow[e] = (uint8_t)h;
    else if (a.cnt_bytes == 2) reinterpret_cast<uint16_t*>(trow)[e] = (uint16_t)h;
    else reinterpret_cast<uint32_t*>(trow)[e] = (uint32_t)h;
  }
  __syncthreads();
  if (threadIdx.x == 0) grid_arrive(a.hdr, (uint32_t)a.G);

  // ---- while the other blocks finish: each selection's rank among this
  //      block's selections of the same expert, in item order (per-warp counts
  //      over a contiguous split of the items, their exclusive prefix over
  //      warps, then a walk that ranks equal experts inside each 32-item chunk)
  const long long i_begin = (long long)t_begin * a.k;
  const int w_begin = (int)((long long)n_items * warp / kWarps);
  const int w_end = (int)((long long)n_items * (warp + 1) / kWarps);
  if (lrank_s) {
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) hist_w[i] = 0;
    __syncthreads();
    for (int i = w_begin + lane; i < w_end; i += 32) {
      const int e = ids_s[i];
      if (e < E) atomicAdd(&hist_w[warp * E + e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int h[kWarps];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) h[w] = hist_w[w * E + e];
      int run = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        hist_w[w * E + e] = run;
        run += h[w];
      }
    }
    __syncthreads();
    for (int i0 = w_begin; i0 < w_end; i0 += 32) {
      // rank inside the 32-item chunk = earlier lanes holding the same expert
      // (inactive lanes hold distinct negative values); the chunk's last item of
      // each expert then raises the running count
      const int i = i0 + lane;
      const bool act = i < w_end;
      const int e = act ? min((int)ids_s[i], E - 1) : -1 - lane;  // ids were range-checked when selected
      int rank = 0;
#pragma unroll
      for (int d = 1; d < 32; ++d) {
        const int o = __shfl_up_sync(0xffffffffu, e, d);
        rank += (lane >= d && o == e) ? 1 : 0;
      }
      int slot = 0;
      if (act) {
        slot = hist_w[warp * E + e] + rank;
        lrank_s[i] = (uint16_t)slot;
      }
      __syncwarp();
      if (act) atomicMax(&hist_w[warp * E + e], slot + 1);
      __syncwarp();
    }
  }
  if (threadIdx.x == 0) flag[0] = grid_wait(a.hdr, (uint32_t)a.G, gen, a.timeout_ns) ? 1 : 0;
  __syncthreads();
  if (!flag[0]) return;
  if (!staged_ok) return;  // a staging wait gave up (recorded); outputs undefined

  // ---------------- phase 2: totals and block base from the table ----------------
  // Every block reads every row of the table: the sum of all rows gives the
  // expert counts, the sum of the rows of earlier blocks this block's base.
  // Thread (row group rg, word w) reads 32-bit word w of rows rg, rg + R, ...
  // (a warp reads consecutive words: coalesced), all loads in flight, and
  // keeps per-entry sums; the partial sums go to shared memory word-major so
  // the stores and the reduction reads hit distinct banks.  Integer sums in a
  // fixed order: deterministic, no atomics.
  int P = 0;
  {
    const int WPR = a.row_stride >> 2;                     // 32-bit words per row
    const int EPW = 4 / a.cnt_bytes;                       // entries per word
    const int R = max(1, min((int)blockDim.x / WPR, a.G));  // row groups
    const int rg = threadIdx.x / WPR, w = threadIdx.x % WPR;
    int tot[4] = {0, 0, 0, 0}, pre[4] = {0, 0, 0, 0};
    const bool wide = a.cnt_bytes == 1 && (a.row_stride >> 4) * 16 <= (int)blockDim.x;
    if (wide) {
      // byte entries, 16-byte loads: thread (row group rg4 < 16, 16-byte column w4)
      // reads rows rg4, rg4 + 16, ... (all loads in flight) and keeps two 16-bit
      // lanes per 32-bit accumulator (a row group's sums stay below 65536)
      const int W4 = a.row_stride >> 4;
      const int R4 = min(16, a.G);
      const int rg4 = threadIdx.x / W4, w4 = threadIdx.x % W4;
      uint32_t* part_w = reinterpret_cast<uint32_t*>(stage);  // [2][R4][8][W4 + 1] packed pairs
      const int pstride = W4 + 1;
      if (rg4 < R4) {
        uint32_t acc_t[8] = {0, 0, 0, 0, 0, 0, 0, 0}, acc_p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        constexpr int kB4 = 10;
        for (int cp0 = rg4; cp0 < a.G; cp0 += R4 * kB4) {
          uint4 v[kB4];
#pragma unroll
          for (int b = 0; b < kB4; ++b) {
            const int cp = cp0 + b * R4;
            v[b] = cp < a.G ? __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(a.table) +
                                                                     (size_t)cp * a.row_stride) + w4)
                            : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int b = 0; b < kB4; ++b) {
            const bool before = cp0 + b * R4 < c;
            const uint32_t vw[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t e02 = vw[j] & 0x00ff00ffu, e13 = (vw[j] >> 8) & 0x00ff00ffu;
              acc_t[2 * j] += e02;
              acc_t[2 * j + 1] += e13;
              if (before) {
                acc_p[2 * j] += e02;
                acc_p[2 * j + 1] += e13;
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          part_w[(rg4 * 8 + j) * pstride + w4] = acc_t[j];
          part_w[((R4 + rg4) * 8 + j) * pstride + w4] = acc_p[j];
        }
      }
      __syncthreads();
      // entry e = 16*w4 + 4*j + lo/hi*2 + odd: accumulator 2*j + odd, 16-bit lane lo/hi
      for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int ww = e >> 4, within = e & 15;
        const int acc = (within >> 2) * 2 + (within & 1), sh = (within & 2) ? 16 : 0;
        int st = 0, sp = 0;
        for (int r = 0; r < R4; ++r) {
          st += (int)((part_w[(r * 8 + acc) * pstride + ww] >> sh) & 0xffffu);
          sp += (int)((part_w[((R4 + r) * 8 + acc) * pstride + ww] >> sh) & 0xffffu);
        }
        cnt[e] = is_local(a, e) ? st : 0;  // another shard's expert: zero width
        hist_cta[e] = sp;
      }
    } else if (rg < R) {
      constexpr int kBatch = 20;
      for (int cp0 = rg; cp0 < a.G; cp0 += R * kBatch) {
        uint32_t v[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int cp = cp0 + b * R;
          v[b] = cp < a.G ? __ldcg(reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(a.table) +
                                                                     (size_t)cp * a.row_stride) + w)
                          : 0u;
        }
        if (a.cnt_bytes == 1) {
          // byte entries: two 16-bit lanes per 32-bit add (entries 0,2 and
          // 1,3); totals stay below 65536 because a block holds <= 255 tokens
          uint32_t t02 = 0, t13 = 0, p02 = 0, p13 = 0;
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const uint32_t e02 = v[b] & 0x00ff00ffu, e13 = (v[b] >> 8) & 0x00ff00ffu;
            t02 += e02;
            t13 += e13;
            if (cp0 + b * R < c) {
              p02 += e02;
              p13 += e13;
            }
          }
          tot[0] += (int)(t02 & 0xffffu); tot[2] += (int)(t02 >> 16);
          tot[1] += (int)(t13 & 0xffffu); tot[3] += (int)(t13 >> 16);
          pre[0] += (int)(p02 & 0xffffu); pre[2] += (int)(p02 >> 16);
          pre[1] += (int)(p13 & 0xffffu); pre[3] += (int)(p13 >> 16);
        } else {
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const bool before = cp0 + b * R < c;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (i < EPW) {
                const int x = a.cnt_bytes == 2 ? (int)((v[b] >> (16 * i)) & 0xffffu) : (int)v[b];
                tot[i] += x;
                pre[i] += before ? x : 0;
              }
            }
          }
        }
      }
    }
    int* part_t = reinterpret_cast<int*>(stage);   // [R][EPW][WPR]
    int* part_p = part_t + R * EPW * WPR;          // [R][EPW][WPR]
    if (!wide && rg < R) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < EPW) {
          part_t[(rg * EPW + i) * WPR + w] = tot[i];
          part_p[(rg * EPW + i) * WPR + w] = pre[i];
        }
    }
    __syncthreads();
    for (int x = threadIdx.x; !wide && x < EPW * WPR; x += blockDim.x) {
      const int i = x / WPR, ww = x % WPR;
      const int e = ww * EPW + i;
      if (e < E) {
        int st = 0, sp = 0;
        for (int r = 0; r < R; ++r) {
          st += part_t[(r * EPW + i) * WPR + ww];
          sp += part_p[(r * EPW + i) * WPR + ww];
        }
        cnt[e] = is_local(a, e) ? st : 0;  // another shard's expert: zero width
        hist_cta[e] = sp;
      }
    }
    if (!lrank_s)
      for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) hist_w[i] = 0;
    __syncthreads();
    scan_padded_offsets(cnt, offs, E, a.tile, scan_scratch);
    P = offs[E];
    if (c == 0) {
      // the shard's experts (those before it have no rows: offs[loc_off] == 0)
      for (int le = threadIdx.x; le < a.loc_n; le += blockDim.x) {
        a.counts[le] = cnt[a.loc_off + le];
        a.offsets[le] = offs[a.loc_off + le];
      }
      if (threadIdx.x == 0) {
        a.offsets[a.loc_n] = P;
        a.totals[0] = P;
        a.totals[1] = P / a.tile;
      }
    }
  }
  const int ntiles = P / a.tile;

  // ---------------- phase 2: slots in token order ----------------
  if (lrank_s) {
    // slot = expert offset + earlier blocks' selections of the expert + local rank
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
      const int e = ids_s[i];
      if (e >= E) {
        record_bounds(a.hdr);
        continue;
      }
      if (!is_local(a, e)) {  // another shard's expert: no slot
        a.e2p[i_begin + i] = -1;
        continue;
      }
      const int slot = offs[e] + hist_cta[e] + lrank_s[i];
      a.e2p[i_begin + i] = slot;
      // token of item i: t_begin + i / k (i < 2^16, so the multiply-high is exact)
      const int lt = a.k == 1 ? i : (int)__umulhi((uint32_t)i, a.kinv);
      if ((unsigned)slot < (unsigned)a.max_padded) a.p2t[slot] = t_begin + lt;
      else record_bounds(a.hdr);
    }
  } else {
    // per-warp counts over a contiguous split of the block's selections, their
    // exclusive prefix over warps, then a walk that ranks equal experts inside
    // each 32-item chunk (match + popcount)
    for (int i = w_begin + lane; i < w_end; i += 32) {
      const int e = ids_s ? (int)ids_s[i] : a.ids[i_begin + i];
      if ((unsigned)e < (unsigned)E) atomicAdd(&hist_w[warp * E + e], 1); else record_bounds(a.hdr);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int run = offs[e] + hist_cta[e];
      for (int w = 0; w < kWarps; ++w) {
        const int h = hist_w[w * E + e];
        hist_w[w * E + e] = run;
        run += h;
      }
    }
    __syncthreads();
    for (int i0 = w_begin; i0 < w_end; i0 += 32) {
      const int i = i0 + lane;
      const bool act = i < w_end;
      const unsigned amask = __ballot_sync(0xffffffffu, act);
      if (act) {
        int e = ids_s ? (int)ids_s[i] : a.ids[i_begin + i];
        if ((unsigned)e >= (unsigned)E) {
          record_bounds(a.hdr);
          e = 0;
        }
        const unsigned m = __match_any_sync(amask, e);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int leader = __ffs(m) - 1;
        const int slot = hist_w[warp * E + e] + rank;
        __syncwarp(amask);
        if (lane == leader) hist_w[warp * E + e] += __popc(m);
        if (is_local(a, e)) {
          a.e2p[i_begin + i] = slot;
          if ((unsigned)slot < (unsigned)a.max_padded) a.p2t[slot] = (int)((i_begin + i) / a.k); else record_bounds(a.hdr);
        } else {
          a.e2p[i_begin + i] = -1;  // another shard's expert: no slot
        }
      }
      __syncwarp();
    }
  }

  // ---------------- tile tables and padding rows (a warp per tile) ----------------
  if (ntiles > a.max_tiles || P > a.max_padded) {
    if (threadIdx.x == 0) record_bounds(a.hdr);
    return;
  }
  const int tc0 = (int)((long long)ntiles * c / a.G), tc1 = (int)((long long)ntiles * (c + 1) / a.G);
  for (int tc = tc0 + warp; tc < tc1; tc += kWarps) {
    const int row = tc * a.tile;
    int lo = 0, hi = E - 1;  // largest e with offs[e] <= row
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (offs[mid] <= row) lo = mid; else hi = mid - 1;
    }
    const int lim = min(row + a.tile, offs[lo] + cnt[lo]);
    if (lane == 0) {
      a.tile_expert[tc] = lo - a.loc_off;  // the local expert (batch index)
      a.tile_mn[tc] = lim;
    }
    for (int r = lim + lane; r < row + a.tile; r += 32) a.p2t[r] = -1;
  }

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
  if (p->num_experts > MOE_MAX_EXPERTS || p->top_k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  const long long items = (long long)p->num_tokens * p->top_k;
  if (items + std::min<long long>(p->num_experts, items) * (p->tile_tokens_dim - 1) > 0x7fffffffLL)
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

int grid_for(const moe_route_params* p, const DevInfo& d) {
  const int T = p->num_tokens;
  int g = (T + 63) / 64;
  g = std::max(1, std::min(g, d.sms));
  return g;
}

// workspace: header | table [G][row] (256-byte aligned, rows sized for the
// widest 4-byte entries; read as 32-bit words)
size_t table_offset(int) { return 256; }

size_t ws_bytes_for(int E, int G) {
  const size_t row = ((size_t)E * 4 + 15) & ~(size_t)15;
  return table_offset(E) + (size_t)G * row;
}

// sigmoid fast path: 8 lanes per token, one lane per E/8 experts
bool fast_path_ok(const moe_route_params* p) {
  if (p->score_fn != MOE_SIGMOID || !p->softmax_before_topk) return false;
  if (p->num_experts % 8 != 0) return false;
  const int V = p->num_experts / 8;
  const bool v_ok = p->logits_dtype == MOE_BF16 ? (V == 8 || V == 16 || V == 32) : (V == 8 || V == 16);
  if (!v_ok) return false;
  const bool grouped = p->n_group > 1 && p->topk_group > 0;
  if (grouped && (p->n_group != 8 || p->group_score_topn > 2)) return false;
  return p->top_k <= 32;
}

template <int VPL, int FAST_ESZ>
cudaError_t launch_route(const RouteArgs& a, int smem, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel<VPL, FAST_ESZ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kStageBytesMax + 128 * 1024);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.G);
  cfg.blockDim = dim3((FAST_ESZ > 0) ? kThreadsFast : kThreadsGeneric);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, route_kernel<VPL, FAST_ESZ>, a);
  if (e != cudaSuccess) {
    // the pair of attributes was refused: a plain cooperative launch
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, route_kernel<VPL, FAST_ESZ>, a);
  }
  return e;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" int moe_route_capacity(const moe_route_params* p, int64_t* max_padded, int64_t* max_tiles) {
  const int v = validate(p);
  if (v != MOE_OK) return v;
  if (!max_padded || !max_tiles) return MOE_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)p->num_tokens * p->top_k;
  const int64_t nz = std::min<int64_t>(rows, p->num_experts);
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
  *bytes = ws_bytes_for(p->num_experts, d.sms);
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
  if (!ws || ws_bytes < ws_bytes_for(p->num_experts, d.sms)) return MOE_ERR_WORKSPACE;

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
  a.table = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(ws) + table_offset(p->num_experts));
  if ((reinterpret_cast<uintptr_t>(ws) & 15) != 0) return MOE_ERR_WORKSPACE;
  a.T = T;
  a.E = p->num_experts;
  a.k = p->top_k;
  a.score_fn = p->score_fn;
  a.pre = p->softmax_before_topk ? 1 : 0;
  a.grouped = (p->n_group > 1 && p->topk_group > 0) ? 1 : 0;
  a.n_group = p->n_group;
  a.topk_group = std::min(p->topk_group, p->n_group);
  a.topn = p->group_score_topn;
  a.renorm = p->renormalize ? 1 : 0;
  a.scale = p->scaling_factor;
  a.tile = p->tile_tokens_dim;
  a.kinv = p->top_k > 1 ? (uint32_t)((0x100000000ull + (uint64_t)p->top_k - 1) / (uint64_t)p->top_k) : 0u;
  a.logits_dtype = p->logits_dtype;
  a.bias_dtype = p->bias_dtype;
  a.weights_dtype = p->weights_dtype;
  a.has_bias = bias != nullptr;
  a.G = grid_for(p, d);
  {
    int64_t mp = 0, mt = 0;
    moe_route_capacity(p, &mp, &mt);
    a.max_padded = (int)mp;
    a.max_tiles = (int)mt;
  }
  a.loc_off = p->local_expert_offset;
  a.loc_n = p->local_num_experts > 0 ? p->local_num_experts : p->num_experts;
  a.row_bytes = p->num_experts * esize(p->logits_dtype);
  const int per_block = (T + a.G - 1) / a.G;
  a.chunk_tokens = std::max(1, std::min(per_block, kStageBytesMax / a.row_bytes));
  a.cnt_bytes = per_block <= 255 ? 1 : (per_block <= 65535 ? 2 : 4);
  a.row_stride = (p->num_experts * a.cnt_bytes + 15) & ~15;
  a.fast = fast_path_ok(p) ? 1 : 0;
  a.timeout_ns = kDefaultTimeoutNs;
  const int nthreads = a.fast ? kThreadsFast : kThreadsGeneric;
  // the stage region also holds phase 2's per-row-group partial sums (two sets)
  const int wpr = a.row_stride / 4;
  const int part_bytes = 2 * std::max(1, std::min(nthreads / wpr, a.G)) * (4 / a.cnt_bytes) * wpr * 4;
  a.stage_bytes = (std::max(a.chunk_tokens * a.row_bytes, part_bytes) + 15) & ~15;
  a.ids_in_smem = ((long long)per_block * a.k * 2 <= 32 * 1024) ? 1 : 0;
  const bool lut = a.fast && p->logits_dtype == MOE_BF16;
  const RouteSmem L = route_smem_layout(a.E, a.stage_bytes, a.ids_in_smem ? per_block * a.k * 2 : 0, nthreads / 32,
                                        lut ? kLutEntries * 4 : 0);
  const int smem = L.total;
  if (smem > d.smem_optin || smem > kStageBytesMax + 128 * 1024) return MOE_ERR_UNSUPPORTED;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (a.fast) {
    const int V = a.E / 8;
    if (p->logits_dtype == MOE_BF16)
      err = V == 8 ? launch_route<8, 2>(a, smem, st) : V == 16 ? launch_route<16, 2>(a, smem, st)
                                                              : launch_route<32, 2>(a, smem, st);
    else
      err = V == 8 ? launch_route<8, 4>(a, smem, st) : launch_route<16, 4>(a, smem, st);
  } else {
    switch (mode) {
      case 0: err = launch_route<0, 0>(a, smem, st); break;
      case 2: err = launch_route<2, 0>(a, smem, st); break;
      case 3: err = launch_route<3, 0>(a, smem, st); break;
      case 4: err = launch_route<4, 0>(a, smem, st); break;
      case 5: err = launch_route<5, 0>(a, smem, st); break;  // e.g. 160 experts in groups of 20
      case 6: err = launch_route<6, 0>(a, smem, st); break;
      case 8: err = launch_route<8, 0>(a, smem, st); break;
      case 12: err = launch_route<12, 0>(a, smem, st); break;
      case 16: err = launch_route<16, 0>(a, smem, st); break;
      case 24: err = launch_route<24, 0>(a, smem, st); break;
      case 32: err = launch_route<32, 0>(a, smem, st); break;
      default: return MOE_ERR_UNSUPPORTED;
    }
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// barrier test hook: a grid that waits for more arrivals than it has blocks
// ---------------------------------------------------------------------------
namespace moe {
namespace {
__global__ void barrier_probe_kernel(WsHeader* hdr, uint32_t expected, long long timeout_ns) {
  __shared__ int flag;
  const uint32_t gen = barrier_generation(hdr);
  grid_barrier(hdr, expected, gen, timeout_ns, &flag);
}
}  // namespace
}  // namespace moe

extern "C" int moe_debug_barrier_wait(int32_t blocks, int32_t extra_arrivals, int64_t timeout_ns, void* ws,
                                      size_t ws_bytes, void* stream) {
  if (blocks <= 0 || extra_arrivals < 0 || timeout_ns <= 0 || timeout_ns > 5LL * 1000 * 1000 * 1000)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  const DevInfo d = device_info();
  if (blocks > d.sms) return MOE_ERR_INVALID_ARG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(32);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, barrier_probe_kernel, hdr,
                                           (uint32_t)(blocks + extra_arrivals), (long long)timeout_ns);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// proxy error hook
// ---------------------------------------------------------------------------
namespace moe {
namespace {
__global__ void proxy_error_kernel(const float* x, long long n, float* out) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = x[i];
    out[i] = fmaf(0.5f, tanh_approx(0.5f * v), 0.5f) - sigmoid_f32(v);
  }
}
}  // namespace
}  // namespace moe

extern "C" int moe_debug_sigmoid_proxy_error(const float* x, int64_t n, float* out, void* stream) {
  if (n < 0 || (n > 0 && (!x || !out))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
  proxy_error_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, (long long)n, out);
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
// first successful set-up also zero-fills the array's 64-byte header on the
// caller's stream; after that the status word is sticky across calls (a
// recorded error stays until moe_route_no_alloc_status clears it).
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
  if (cudaMemsetAsync(p, 0, sizeof(WsHeader), st) != cudaSuccess) return nullptr;
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
  if (ws_bytes_for(p->num_experts, d.sms) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
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
