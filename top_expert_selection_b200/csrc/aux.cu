// Aux-loss path: scores + routing map, load-balancing loss, and its backward.
//
// Sources: Implementation:NVIDIA TransformerEngine Fused Router -- Description
// (fused_compute_score_for_moe_aux_loss: scores and routing map;
// fused_moe_aux_loss: loss from probs and tokens_per_expert; forward and
// backward), Signature (probs, tokens_per_expert, total_num_tokens,
// num_experts, topk, coeff).
//
// loss = coeff * E / (T_total * k) * sum_e (sum_t probs[t,e]) * tpe[e]
//      = C * sum_t sum_e probs[t,e] * tpe[e]
// computed in one pass over probs (no column-sum intermediate).
//
// Determinism: tokens_per_expert is an integer sum (order-free).  The loss is
// reduced from per-thread fp32 partials to per-block double partials over a
// fixed grid, and the last block to finish adds the block partials in index
// order, so the result does not depend on scheduling.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kAuxThreads = 256;
constexpr int kAuxWarps = kAuxThreads / 32;
constexpr int kLossBlocks = 148;  // fixed: one per SM on a 148-SM part; the reduction order depends on it
constexpr int kLossThreads = 512;  // loss forward block (measured faster than 2 x 256 per SM)

// workspace layout after the 64-byte header
struct AuxWs {
  int32_t* tpe_acc;    // [E] running integer counts
  double* partials;    // [kLossBlocks]
};

__host__ __device__ inline size_t aux_ws_bytes(int E) {
  return sizeof(WsHeader) + (((size_t)E * 4 + 255) & ~(size_t)255) + (size_t)kLossBlocks * sizeof(double);
}

__device__ inline AuxWs aux_ws(void* ws, int E) {
  AuxWs w;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws) + sizeof(WsHeader);
  w.tpe_acc = reinterpret_cast<int32_t*>(base);
  w.partials = reinterpret_cast<double*>(base + (((size_t)E * 4 + 255) & ~(size_t)255));
  return w;
}

__device__ __forceinline__ float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

// --------------------------------------------------------------------------
// scores: warp per token, lane l owns experts [l*VPL, l*VPL + VPL)
// --------------------------------------------------------------------------
constexpr int kScoreThreads = 512;

// Top-k mask of one row held by a warp (lane l: entries [l*VPL, l*VPL+VPL)),
// for k <= 8, by threshold and counting instead of k argmax rounds.  In each
// 8-lane group the second-largest lane maximum is at most its group's top-2
// lane maxima, so at least 8 >= k entries are >= tau = the smallest of the
// four groups' second maxima.  The entries >= tau (the candidates) are ranked by
// counting on packed (ordered key, ~index) words - larger value first, equal
// values by lower index - and the mask keeps those at or above the k-th.
// Returns false (warp-uniform) when the candidates exceed 32 or number fewer
// than k (non-finite values); the caller then uses the k rounds.
template <int VPL>
__device__ __forceinline__ bool topk_mask_by_threshold(const float* p, uint32_t valid, int lane, int k,
                                                       unsigned long long* list, uint32_t* chosen_out) {
  const unsigned FULL = 0xffffffffu;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if ((valid >> i) & 1u) mx = fmaxf(mx, p[i]);
  float a1 = mx, a2 = -INFINITY;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    const float o1 = __shfl_xor_sync(FULL, a1, off), o2 = __shfl_xor_sync(FULL, a2, off);
    a2 = fmaxf(fminf(a1, o1), fmaxf(a2, o2));
    a1 = fmaxf(a1, o1);
  }
  float tau = fminf(a2, __shfl_xor_sync(FULL, a2, 8));
  tau = fminf(tau, __shfl_xor_sync(FULL, tau, 16));
  uint32_t cm = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) cm |= (((valid >> i) & 1u) && p[i] >= tau ? 1u : 0u) << i;
  const int cnt = __popc(cm);
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(FULL, incl, off);
    if (lane >= off) incl += o;
  }
  const int total = __shfl_sync(FULL, incl, 31);
  if (total > 32 || total < k) return false;
  int pos = incl - cnt;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if ((cm >> i) & 1u) list[pos++] = pack_key(p[i], lane * VPL + i);
  __syncwarp();
  unsigned long long key = 0ull;
  int rank = 32;
  if (lane < total) {
    key = list[lane];
    rank = 0;
    for (int j = 0; j < total; ++j) rank += (list[j] > key) ? 1 : 0;
  }
  const int src = __ffs(__ballot_sync(FULL, rank == k - 1)) - 1;  // keys are distinct: one lane
  const unsigned long long kth = shfl_xor_u64(FULL, key, src ^ lane);
  uint32_t chosen = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if ((cm >> i) & 1u) chosen |= (pack_key(p[i], lane * VPL + i) >= kth ? 1u : 0u) << i;
  __syncwarp();  // the list is reused by the next row
  *chosen_out = chosen;
  return true;
}

// One row by a whole warp (lane l: entries [l*VPL, l*VPL+VPL)): scores, the
// top-k mask, probs and routing-map stores, the mask counted into hist.
template <int VPL>
__device__ __forceinline__ void score_row_warp(long long t, int E, int k, int score_fn, const float* __restrict__ logits,
                                               float* __restrict__ probs, uint8_t* __restrict__ rmap, int* hist,
                                               unsigned long long* list, int lane) {
  const unsigned FULL = 0xffffffffu;
  uint32_t valid = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) valid |= ((lane * VPL + i < E) ? 1u : 0u) << i;
  // a lane's VPL experts are contiguous: 16-byte loads when the row allows it
  const bool vec = (VPL % 4 == 0) && ((E & 3) == 0) && (lane * VPL + VPL <= E);
  float x[VPL], p[VPL];
  {
    const float* row = logits + t * E;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec) {
        if ((i & 3) == 0) {
          const float4 q = __ldcs(reinterpret_cast<const float4*>(row + e));
          x[i] = q.x;
          if (i + 1 < VPL) x[i + 1] = q.y;
          if (i + 2 < VPL) x[i + 2] = q.z;
          if (i + 3 < VPL) x[i + 3] = q.w;
        }
      } else {
        x[i] = e < E ? __ldcs(row + e) : 0.0f;
      }
    }
  }
  float sum = 0.0f;
  if (score_fn == MOE_SOFTMAX) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (valid & (1u << i)) m = fmaxf(m, x[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      p[i] = (valid & (1u << i)) ? expf(x[i] - m) : 0.0f;
      sum += p[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      p[i] = (valid & (1u << i)) ? sigmoid_f32(x[i]) : 0.0f;
      sum += p[i];
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
#pragma unroll
  for (int i = 0; i < VPL; ++i) p[i] = p[i] / sum;

  // top-k mask over probs, ties -> lower expert: threshold + counting, else
  // k rounds of warp argmax
  uint32_t avail = valid, chosen = 0;
  bool done = false;
  if constexpr (VPL <= 8) {
    if (k <= 8) done = topk_mask_by_threshold<VPL>(p, valid, lane, k, list, &chosen);
  }
  for (int j = 0; j < k && !done; ++j) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (avail & (1u << i)) {
        const unsigned long long pk = pack_key(p[i], lane * VPL + i);
        best = pk > best ? pk : best;
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const unsigned long long o = shfl_xor_u64(FULL, best, off);
      best = o > best ? o : best;
    }
    const int win = packed_expert(best);
    if (win / VPL == lane) {
      const uint32_t bit = 1u << (win - lane * VPL);
      avail &= ~bit;
      chosen |= bit;
    }
  }
  float* prow = probs + t * E;
  uint8_t* mrow = rmap + t * E;
  if constexpr (VPL % 4 == 0) {
    if (vec) {
#pragma unroll
      for (int i = 0; i < VPL; i += 4) {
        const int e = lane * VPL + i;
        __stcs(reinterpret_cast<float4*>(prow + e), make_float4(p[i], p[i + 1], p[i + 2], p[i + 3]));
        const uint32_t m4 = ((chosen >> i) & 1u) | (((chosen >> (i + 1)) & 1u) << 8) |
                            (((chosen >> (i + 2)) & 1u) << 16) | (((chosen >> (i + 3)) & 1u) << 24);
        *reinterpret_cast<uint32_t*>(mrow + e) = m4;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if ((chosen >> i) & 1u) atomicAdd(&hist[lane * VPL + i], 1);
      return;
    }
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane * VPL + i;
    if (valid & (1u << i)) {
      __stcs(prow + e, p[i]);
      const bool c = (chosen >> i) & 1u;
      mrow[e] = c ? 1 : 0;
      if (c) atomicAdd(&hist[e], 1);
    }
  }
}

// The block's counts into the accumulator; the last block to finish publishes
// them to tokens_per_expert and clears the accumulator.
// The block's atomics are ordered before its ticket by the barrier and thread
// 0's fence (a fence orders what its thread has observed, which the barrier
// makes the other threads' atomics); the other threads do not fence, so they
// do not wait for their own probs and routing-map stores to drain.
__device__ __forceinline__ void publish_counts(int E, const int* hist, int32_t* __restrict__ tpe, void* ws) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  AuxWs w = aux_ws(ws, E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(&w.tpe_acc[e], hist[e]);
  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = (atomicAdd(&hdr->ticket, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (last) {
    __threadfence();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      tpe[e] = __ldcg(&w.tpe_acc[e]);
      w.tpe_acc[e] = 0;
    }
    if (threadIdx.x == 0) hdr->ticket = 0;
  }
}

template <int VPL>
__global__ void __launch_bounds__(kScoreThreads, 3) aux_scores_kernel(int T, int E, int k, int score_fn,
                                                                 const float* __restrict__ logits,
                                                                 float* __restrict__ probs,
                                                                 uint8_t* __restrict__ rmap,
                                                                 int32_t* __restrict__ tpe, void* ws) {
  extern __shared__ int hist[];  // [E], then per warp 32 packed candidate keys
  pdl_entry();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  unsigned long long* list = reinterpret_cast<unsigned long long*>(hist + ((E + 1) & ~1)) + warp * 32;
  for (long long t = (long long)blockIdx.x * nw + warp; t < T; t += (long long)gridDim.x * nw)
    score_row_warp<VPL>(t, E, k, score_fn, logits, probs, rmap, hist, list, lane);
  publish_counts(E, hist, tpe, ws);
}

// --------------------------------------------------------------------------
// scores, four tokens per warp (E = 8V, k <= 8): the 8 lanes of group g take
// token 4q + g; lane j holds experts c*32 + 4j + r (c < V/4, r < 4), so each
// 16-byte load or store of a chunk c covers 128 contiguous bytes of the row.
//
// Top-k mask without k argmax rounds: every lane keeps the three largest of
// its V probs; k extraction rounds over those lists (each round the group's
// largest head is popped) give a value tau with at least k entries >= tau
// (the k popped ones), so the entries >= tau include the top k.  The head
// keys carry the lane in their 3 low bits so that one head is popped per
// round; tau is the k-th popped key with those bits cleared, which is at most
// the popped entries' values.  When exactly k entries are >= tau, they are
// the mask; otherwise (a lane held more than three of the top k, or ties)
// the least candidate -- smallest prob, then highest expert -- is dropped
// until k remain.  A row whose score sum is not finite is redone by the whole
// warp with the per-row path above.
// --------------------------------------------------------------------------
constexpr int kQuadThreads = 256;

template <int V>
__device__ __noinline__ void score_row_warp_out_of_line(long long t, int k, int score_fn, const float* logits,
                                                        float* probs, uint8_t* rmap, int* hist,
                                                        unsigned long long* list, int lane) {
  score_row_warp<V / 4>(t, 8 * V, k, score_fn, logits, probs, rmap, hist, list, lane);
}

template <int V>
__global__ void __launch_bounds__(kQuadThreads, V >= 32 ? 2 : 3) aux_scores_quad_kernel(int T, int k, int score_fn,
                                                                      const float* __restrict__ logits,
                                                                      float* __restrict__ probs,
                                                                      uint8_t* __restrict__ rmap,
                                                                      int32_t* __restrict__ tpe, void* ws) {
  constexpr int E = 8 * V, NC = V / 4;
  extern __shared__ int hist[];  // [E], then per warp 32 keys for the per-row path
  const unsigned FULL = 0xffffffffu;
  pdl_entry();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 3, j = lane & 7;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  unsigned long long* list = reinterpret_cast<unsigned long long*>(hist + E) + warp * 32;

  // routing-map bytes of this lane's experts summed over its tokens, 4 per word
  uint32_t cnt4[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) cnt4[c] = 0u;
  auto flush = [&]() {  // 4 groups x at most 63 tokens per byte: no carry
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      uint32_t v = cnt4[c];
      v += __shfl_xor_sync(FULL, v, 8);
      v += __shfl_xor_sync(FULL, v, 16);
      if (g == 0 && v) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int n = (v >> (8 * r)) & 255;
          if (n) atomicAdd(&hist[c * 32 + 4 * j + r], n);
        }
      }
      cnt4[c] = 0u;
    }
  };

  const long long nq = ((long long)T + 3) >> 2;
  const long long qstride = (long long)gridDim.x * nw;
  int since_flush = 0;
  // the next group's rows are loaded while this one is scored
  float4 nx[NC];
  auto load_quad = [&](long long qq) {
    const long long tt = 4 * qq + g;
    const float* row = logits + tt * E + 4 * j;
#pragma unroll
    for (int c = 0; c < NC; ++c)
      nx[c] = (qq < nq && tt < T) ? __ldcs(reinterpret_cast<const float4*>(row + c * 32))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  load_quad((long long)blockIdx.x * nw + warp);
  for (long long q = (long long)blockIdx.x * nw + warp; q < nq; q += qstride) {
    const long long t = 4 * q + g;
    const bool tv = t < T;
    float p[V];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      p[4 * c] = nx[c].x;
      p[4 * c + 1] = nx[c].y;
      p[4 * c + 2] = nx[c].z;
      p[4 * c + 3] = nx[c].w;
    }
    load_quad(q + qstride);
    float sum = 0.0f;
    if (score_fn == MOE_SOFTMAX) {
      float m = p[0];
#pragma unroll
      for (int i = 1; i < V; ++i) m = fmaxf(m, p[i]);
      m = fmaxf(m, __shfl_xor_sync(FULL, m, 1));
      m = fmaxf(m, __shfl_xor_sync(FULL, m, 2));
      m = fmaxf(m, __shfl_xor_sync(FULL, m, 4));
#pragma unroll
      for (int i = 0; i < V; ++i) {
        p[i] = expf(p[i] - m);
        sum += p[i];
      }
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        p[i] = sigmoid_f32(p[i]);
        sum += p[i];
      }
    }
    sum += __shfl_xor_sync(FULL, sum, 1);
    sum += __shfl_xor_sync(FULL, sum, 2);
    sum += __shfl_xor_sync(FULL, sum, 4);
    // p / sum: one reciprocal per row and two corrections per entry give the
    // IEEE quotient; rows with an entry or sum outside that method's range
    // divide directly
    {
      bool direct = !(sum >= kDivMinDen && sum <= kDivMaxDen);
#pragma unroll
      for (int i = 0; i < V; ++i) direct |= p[i] < kDivMinNum;
      if (__any_sync(FULL, direct)) {
#pragma unroll
        for (int i = 0; i < V; ++i) p[i] = p[i] / sum;
      } else {
        const float y = 1.0f / sum;
#pragma unroll
        for (int i = 0; i < V; ++i) p[i] = div_rn_by_recip(p[i], sum, y);
      }
    }
    const bool hard = tv && !isfinite(sum);  // group-uniform
    const bool fast = tv && !hard;

    // the three largest probs of this lane (fast rows: every prob >= 0)
    float a1 = -1.0f, a2 = -1.0f, a3 = -1.0f;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      a3 = fmaxf(a3, fminf(a2, p[i]));
      a2 = fmaxf(a2, fminf(a1, p[i]));
      a1 = fmaxf(a1, p[i]);
    }
    const uint32_t tag = 7u - (uint32_t)j;  // distinct per lane of a group
    uint32_t h1 = (__float_as_uint(a1) & ~7u) | tag, h2 = (__float_as_uint(a2) & ~7u) | tag,
             h3 = (__float_as_uint(a3) & ~7u) | tag, mx = 0u;
    for (int r = 0; r < k; ++r) {
      mx = h1;
      mx = max(mx, __shfl_xor_sync(FULL, mx, 1));
      mx = max(mx, __shfl_xor_sync(FULL, mx, 2));
      mx = max(mx, __shfl_xor_sync(FULL, mx, 4));
      const bool win = h1 == mx;
      h1 = win ? h2 : h1;
      h2 = win ? h3 : h2;
      h3 = win ? 0u : h3;
    }
    const float tau = __uint_as_float(mx & ~7u);
    uint32_t cm = 0u;
#pragma unroll
    for (int i = 0; i < V; ++i) cm |= (p[i] >= tau ? 1u : 0u) << i;
    int cnt = __popc(cm);
    cnt += __shfl_xor_sync(FULL, cnt, 1);
    cnt += __shfl_xor_sync(FULL, cnt, 2);
    cnt += __shfl_xor_sync(FULL, cnt, 4);
    int excess = fast ? cnt - k : 0;  // >= 0; group-uniform
    while (__any_sync(FULL, excess > 0)) {
      // drop the group's least candidate: smallest prob, then highest expert
      unsigned long long lk = ~0ull;
      int li = 0;
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const unsigned long long key =
            ((unsigned long long)__float_as_uint(p[i]) << 32) | (uint32_t)(0xffff - ((i >> 2) * 32 + 4 * j + (i & 3)));
        if (((cm >> i) & 1u) && key < lk) {
          lk = key;
          li = i;
        }
      }
      unsigned long long gk = lk;
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        const unsigned long long o = shfl_xor_u64(FULL, gk, off);
        gk = o < gk ? o : gk;
      }
      if (excess > 0 && lk == gk) cm &= ~(1u << li);
      excess -= excess > 0 ? 1 : 0;
    }
    if (fast) {
      float* prow = probs + t * E + 4 * j;
      uint8_t* mrow = rmap + t * E + 4 * j;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        __stcs(reinterpret_cast<float4*>(prow + c * 32), make_float4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]));
        const uint32_t b = (((cm >> (4 * c)) & 15u) * 0x00204081u) & 0x01010101u;  // bit r -> byte r
        __stcs(reinterpret_cast<unsigned int*>(mrow + c * 32), b);
        cnt4[c] += b;
      }
    }
    // rows with a non-finite sum: the whole warp, one row at a time
    for (uint32_t hb = __ballot_sync(FULL, hard && j == 0); hb; hb &= hb - 1) {
      const int gg = (__ffs(hb) - 1) >> 3;
      score_row_warp_out_of_line<V>(4 * q + gg, k, score_fn, logits, probs, rmap, hist, list, lane);
    }
    if (++since_flush == 63) {
      flush();
      since_flush = 0;
    }
  }
  flush();
  publish_counts(E, hist, tpe, ws);
}

// --------------------------------------------------------------------------
// loss forward: one pass over probs; fixed grid; deterministic reduction
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(kLossThreads, 1) aux_loss_fwd_kernel(long long n, int E, double C,
                                                                   const float* __restrict__ probs,
                                                                   const int32_t* __restrict__ tpe, float* loss,
                                                                   void* ws) {
  extern __shared__ float tpe_s[];  // [E]
  __shared__ double red[kLossThreads / 32];
  pdl_entry();
  __shared__ int last;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  AuxWs w = aux_ws(ws, E);
  // each block owns a contiguous range of elements (whole rows when E is a
  // multiple of 4); threads stride through it
  const long long rows = n / E;
  const long long per = (E & 3) == 0 ? ((rows + gridDim.x - 1) / gridDim.x) * E
                                     : (((n + gridDim.x - 1) / gridDim.x) + 3) & ~3LL;  // float4 ranges
  const long long b0 = (long long)blockIdx.x * per, b1 = min(n, b0 + per);
  float acc = 0.0f;
  if ((E & 3) == 0 && ((blockDim.x * 4) % (unsigned)E) == 0 && (reinterpret_cast<uintptr_t>(tpe) & 15) == 0) {
    // every float4 a thread loads covers the same four columns: sum the
    // float4s, then one dot product with those columns' counts
    const long long q1 = b1 >> 2;
    const float4* base = reinterpret_cast<const float4*>(probs) + (b0 >> 2);
    const int nq = (int)(q1 - (b0 >> 2));
    constexpr int kB = 16;
    float4 v[kB];
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      const int l = threadIdx.x + b * (int)blockDim.x;
      v[b] = l < nq ? __ldcs(base + l) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int e = (int)((threadIdx.x * 4) % (unsigned)E);
    const int4 c4 = __ldg(reinterpret_cast<const int4*>(tpe + e));
    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int b = 0; b < kB; ++b) {
      s4.x += v[b].x;
      s4.y += v[b].y;
      s4.z += v[b].z;
      s4.w += v[b].w;
    }
    for (int l = threadIdx.x + kB * (int)blockDim.x; l < nq; l += (int)blockDim.x) {
      const float4 u = __ldcs(base + l);
      s4.x += u.x;
      s4.y += u.y;
      s4.z += u.z;
      s4.w += u.w;
    }
    acc = fmaf(s4.x, (float)c4.x, fmaf(s4.y, (float)c4.y, fmaf(s4.z, (float)c4.z, s4.w * (float)c4.w)));
  } else {
  for (int e = threadIdx.x; e < E; e += blockDim.x) tpe_s[e] = (float)tpe[e];
  __syncthreads();
  if ((E & 3) == 0 && (b0 & 3) == 0) {
    const long long q1 = b1 >> 2;
    const float4* base = reinterpret_cast<const float4*>(probs) + (b0 >> 2);
    const int nq = (int)(q1 - (b0 >> 2));  // float4s of this block (< 2^31)
    constexpr int kB = 16;                 // independent 16-byte loads in flight per thread
    // column of a float4: advances by step (mod E) from one load to the next,
    // so the only division is the first one
    const int step = (int)((blockDim.x * 4) % (unsigned)E);
    int e = (int)((((b0 >> 2) + threadIdx.x) << 2) % E);
    for (int l0 = threadIdx.x; l0 < nq; l0 += blockDim.x * kB) {
      float4 v[kB];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int l = l0 + b * (int)blockDim.x;
        v[b] = l < nq ? __ldcs(base + l) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        // entries past the block's range load as zeros and add nothing
        acc = fmaf(v[b].x, tpe_s[e], acc);
        acc = fmaf(v[b].y, tpe_s[e + 1], acc);
        acc = fmaf(v[b].z, tpe_s[e + 2], acc);
        acc = fmaf(v[b].w, tpe_s[e + 3], acc);
        e += step;
        if (e >= E) e -= E;
      }
    }
    for (long long i = (q1 << 2) + threadIdx.x; i < b1; i += blockDim.x) acc = fmaf(probs[i], tpe_s[i % E], acc);
  } else {
    for (long long i = b0 + threadIdx.x; i < b1; i += blockDim.x) acc = fmaf(probs[i], tpe_s[i % E], acc);
  }
  }
  double d = (double)acc;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = d;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kLossThreads / 32; ++i) s += red[i];
    w.partials[blockIdx.x] = s;
    __threadfence();
    last = (atomicAdd(&hdr->ticket, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (last && threadIdx.x < 32) {
    // warp 0 adds the block partials: lane l takes blocks l, l+32, ... (all
    // loads in flight), then a fixed shuffle tree -- the same order every call
    __threadfence();
    double s = 0.0;
    for (unsigned b = threadIdx.x; b < gridDim.x; b += 32) s += __ldcg(&w.partials[b]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (threadIdx.x == 0) {
      *loss = (float)(C * s);
      hdr->ticket = 0;
    }
  }
}

// --------------------------------------------------------------------------
// loss backward: warp per row
// --------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(kAuxThreads) aux_loss_bwd_kernel(int T, int E, float C,
                                                                   const float* __restrict__ grad_loss,
                                                                   const float* __restrict__ probs,
                                                                   const int32_t* __restrict__ tpe,
                                                                   float* __restrict__ grad_probs,
                                                                   float* __restrict__ grad_logits) {
  extern __shared__ float gp_s[];  // [E] = g * C * tpe[e]
  pdl_entry();
  const float g = *grad_loss;
  for (int e = threadIdx.x; e < E; e += blockDim.x) gp_s[e] = g * C * (float)tpe[e];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (long long t = (long long)blockIdx.x * kAuxWarps + warp; t < T; t += (long long)gridDim.x * kAuxWarps) {
    const float* prow = probs + t * E;
    float p[VPL], gp[VPL];
    float dot = 0.0f;
    const bool vec = (VPL % 4 == 0) && ((E & 3) == 0) && (lane * VPL + VPL <= E);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec && (i & 3) == 0) {
        const float4 q = __ldcs(reinterpret_cast<const float4*>(prow + e));
        p[i] = q.x;
        if (i + 1 < VPL) p[i + 1] = q.y;
        if (i + 2 < VPL) p[i + 2] = q.z;
        if (i + 3 < VPL) p[i + 3] = q.w;
      } else if (!vec) {
        p[i] = e < E ? __ldcs(prow + e) : 0.0f;
      }
      gp[i] = e < E ? gp_s[e] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) dot = fmaf(p[i], gp[i], dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec && (i & 3) == 0 && i + 3 < VPL) {
        if (grad_probs)
          __stcs(reinterpret_cast<float4*>(grad_probs + t * E + e), make_float4(gp[i], gp[i + 1], gp[i + 2], gp[i + 3]));
        if (grad_logits)
          __stcs(reinterpret_cast<float4*>(grad_logits + t * E + e),
                 make_float4(p[i] * (gp[i] - dot), p[i + 1] * (gp[i + 1] - dot), p[i + 2] * (gp[i + 2] - dot),
                             p[i + 3] * (gp[i + 3] - dot)));
      } else if (!vec && e < E) {
        if (grad_probs) __stcs(grad_probs + t * E + e, gp[i]);
        if (grad_logits) __stcs(grad_logits + t * E + e, p[i] * (gp[i] - dot));
      }
    }
  }
}

// --------------------------------------------------------------------------
// backward of the softmax scores: warp per row, dot = sum_j p_j g_j (fp32,
// fixed order: lane partials then a shuffle tree), grad = p * (g - dot)
// --------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(kAuxThreads) aux_scores_bwd_kernel(int T, int E, const float* __restrict__ probs,
                                                                     const float* __restrict__ grad_probs,
                                                                     float* __restrict__ grad_logits, bool aligned) {
  pdl_entry();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool vec = aligned && (VPL % 4 == 0) && ((E & 3) == 0) && (lane * VPL + VPL <= E);
  for (long long t = (long long)blockIdx.x * kAuxWarps + warp; t < T; t += (long long)gridDim.x * kAuxWarps) {
    const float* prow = probs + t * E;
    const float* grow = grad_probs + t * E;
    float p[VPL], g[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec) {
        if ((i & 3) == 0) {
          const float4 a = __ldcs(reinterpret_cast<const float4*>(prow + e));
          const float4 b = __ldcs(reinterpret_cast<const float4*>(grow + e));
          p[i] = a.x; g[i] = b.x;
          if (i + 1 < VPL) { p[i + 1] = a.y; g[i + 1] = b.y; }
          if (i + 2 < VPL) { p[i + 2] = a.z; g[i + 2] = b.z; }
          if (i + 3 < VPL) { p[i + 3] = a.w; g[i + 3] = b.w; }
        }
      } else {
        p[i] = e < E ? __ldcs(prow + e) : 0.0f;
        g[i] = e < E ? __ldcs(grow + e) : 0.0f;
      }
    }
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) dot = fmaf(p[i], g[i], dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec) {
        if ((i & 3) == 0 && i + 3 < VPL)
          __stcs(reinterpret_cast<float4*>(grad_logits + t * E + e),
                 make_float4(p[i] * (g[i] - dot), p[i + 1] * (g[i + 1] - dot), p[i + 2] * (g[i + 2] - dot),
                             p[i + 3] * (g[i + 3] - dot)));
      } else if (e < E) {
        __stcs(grad_logits + t * E + e, p[i] * (g[i] - dot));
      }
    }
  }
}

// --------------------------------------------------------------------------
// backward of the scores from the logits (softmax, or sigmoid over the row
// sum): warp per row, the scores recomputed as the forward computes them,
// dot = sum_e p_e g_e (lane partials, then a shuffle tree),
// grad = d * (g - dot) with d = p (softmax) or p * (1 - s) = s (1 - s) / S
// (sigmoid; 1 - s formed as exp(-x) * s, without cancellation)
// --------------------------------------------------------------------------
template <int VPL>
__device__ __forceinline__ void load_row_f32(const float* __restrict__ row, int E, int lane, bool vec, float* v) {
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane * VPL + i;
    if (vec) {
      if ((i & 3) == 0) {
        const float4 q = __ldcs(reinterpret_cast<const float4*>(row + e));
        v[i] = q.x;
        if (i + 1 < VPL) v[i + 1] = q.y;
        if (i + 2 < VPL) v[i + 2] = q.z;
        if (i + 3 < VPL) v[i + 3] = q.w;
      }
    } else {
      v[i] = e < E ? __ldcs(row + e) : 0.0f;
    }
  }
}

template <int VPL>
__global__ void __launch_bounds__(kAuxThreads) aux_scores_bwd_logits_kernel(int T, int E, int score_fn,
                                                                            const float* __restrict__ logits,
                                                                            const float* __restrict__ grad_probs,
                                                                            float* __restrict__ grad_logits,
                                                                            bool aligned) {
  const unsigned FULL = 0xffffffffu;
  pdl_entry();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool vec = aligned && (VPL % 4 == 0) && ((E & 3) == 0) && (lane * VPL + VPL <= E);
  uint32_t valid = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) valid |= ((lane * VPL + i < E) ? 1u : 0u) << i;
  for (long long t = (long long)blockIdx.x * kAuxWarps + warp; t < T; t += (long long)gridDim.x * kAuxWarps) {
    float x[VPL], g[VPL], p[VPL], d[VPL];
    load_row_f32<VPL>(logits + t * E, E, lane, vec, x);
    load_row_f32<VPL>(grad_probs + t * E, E, lane, vec, g);
    float sum = 0.0f;
    if (score_fn == MOE_SOFTMAX) {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (valid & (1u << i)) m = fmaxf(m, x[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        p[i] = (valid & (1u << i)) ? expf(x[i] - m) : 0.0f;
        sum += p[i];
      }
    } else {
      // s = 1 / (1 + u) with u = exp(-x) (the forward's sigmoid); 1 - s = u * s
      // keeps its relative precision where s rounds close to 1 (d[] holds it)
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const float u = expf(-x[i]);
        p[i] = (valid & (1u << i)) ? 1.0f / (1.0f + u) : 0.0f;
        d[i] = p[i] > 0.0f ? u * p[i] : 1.0f;
        sum += p[i];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      p[i] = p[i] / sum;
      d[i] = score_fn == MOE_SOFTMAX ? p[i] : p[i] * d[i];
      dot = fmaf(p[i], g[i], dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(FULL, dot, off);
    float* out = grad_logits + t * E;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane * VPL + i;
      if (vec) {
        if ((i & 3) == 0 && i + 3 < VPL)
          __stcs(reinterpret_cast<float4*>(out + e),
                 make_float4(d[i] * (g[i] - dot), d[i + 1] * (g[i + 1] - dot), d[i + 2] * (g[i + 2] - dot),
                             d[i + 3] * (g[i + 3] - dot)));
      } else if (e < E) {
        __stcs(out + e, d[i] * (g[i] - dot));
      }
    }
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

int pick_vpl(int E) {
  for (int v : {1, 2, 3, 4, 6, 8, 12, 16, 24, 32})
    if (v * 32 >= E) return v;
  return -1;
}

#define MOE_VPL_SWITCH(vpl, KERNEL_CALL) \
  switch (vpl) {                         \
    case 1: { constexpr int V = 1; KERNEL_CALL; } break;  \
    case 2: { constexpr int V = 2; KERNEL_CALL; } break;  \
    case 3: { constexpr int V = 3; KERNEL_CALL; } break;  \
    case 4: { constexpr int V = 4; KERNEL_CALL; } break;  \
    case 6: { constexpr int V = 6; KERNEL_CALL; } break;  \
    case 8: { constexpr int V = 8; KERNEL_CALL; } break;  \
    case 12: { constexpr int V = 12; KERNEL_CALL; } break; \
    case 16: { constexpr int V = 16; KERNEL_CALL; } break; \
    case 24: { constexpr int V = 24; KERNEL_CALL; } break; \
    case 32: { constexpr int V = 32; KERNEL_CALL; } break; \
    default: return MOE_ERR_UNSUPPORTED;  \
  }

}  // namespace
}  // namespace moe

using namespace moe;

// --------------------------------------------------------------------------
// backward of the routed weights: warp per token; lane j < k holds slot j
// (expert, upstream gradient, score); lane l writes row entries
// [l*VPL, l*VPL + VPL).  fp32, fixed reduction orders.
// --------------------------------------------------------------------------
template <int VPL>
__global__ void __launch_bounds__(kAuxThreads) route_weights_bwd_kernel(int T, int E, int k, int score_fn, int pre,
                                                                        int renorm, float scale, const void* logits,
                                                                        int logits_dtype, const int32_t* ids,
                                                                        const float* grad_w, float* grad_logits,
                                                                        WsHeader* hdr) {
  pdl_entry();
  const unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool vec = (VPL % 4 == 0) && ((E & 3) == 0) && (lane * VPL + VPL <= E) &&
                   ((reinterpret_cast<uintptr_t>(grad_logits) & 15) == 0);
  const bool xvec = (VPL % 8 == 0) && logits_dtype == MOE_BF16 && ((E & 7) == 0) && (lane * VPL + VPL <= E) &&
                    ((reinterpret_cast<uintptr_t>(logits) & 15) == 0);
  const bool slot = lane < k;
  // a row's inputs: the slot lanes' ids and weight gradients, and the lane's
  // logits (experts lane*VPL + i); a slot lane later takes its selected
  // logit from the owning lane
  auto load_row = [&](long long t, int& e, float& gw, float* x) {
    e = slot ? ids[t * k + lane] : 0;
    gw = slot ? grad_w[t * k + lane] : 0.0f;
    if (xvec) {
      const uint16_t* xr = reinterpret_cast<const uint16_t*>(logits) + (size_t)t * E + lane * VPL;
#pragma unroll
      for (int i = 0; i < VPL; i += 8) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(xr + i));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          x[i + 2 * h] = __uint_as_float(w[h] << 16);
          x[i + 2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int ee = lane * VPL + i;
        x[i] = ee < E ? load_as_f32(logits, logits_dtype, (size_t)t * E + ee) : -INFINITY;
      }
    }
  };
  const long long stride = (long long)gridDim.x * kAuxWarps;
  long long t = (long long)blockIdx.x * kAuxWarps + warp;
  int e_next = 0;
  float gw_next = 0.0f, x_next[VPL];
  if (t < T) load_row(t, e_next, gw_next, x_next);
  for (; t < T; t += stride) {
    int e = e_next;
    const float gw = gw_next;
    float x[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) x[i] = x_next[i];
    if (t + stride < T) load_row(t + stride, e_next, gw_next, x_next);  // in flight during this row
    if (slot && (unsigned)e >= (unsigned)E) {
      if (hdr) record_bounds(hdr);
      e = 0;
    }
    float xj = -INFINITY;
    {
      const int src = e / VPL, sub = e - src * VPL;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const float o = __shfl_sync(FULL, x[i], src);
        if (i == sub) xj = o;
      }
      if (!slot) xj = -INFINITY;
    }
    // scores of the selected (v) and, for softmax before top-k, of the lane's row entries (p)
    float v = 0.0f, pr[VPL];
    float m = 0.0f, z = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) pr[i] = 0.0f;
    if (score_fn == MOE_SIGMOID) {
      v = slot ? sigmoid_f32(xj) : 0.0f;
    } else if (pre) {
      m = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i) m = fmaxf(m, x[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        pr[i] = lane * VPL + i < E ? expf(x[i] - m) : 0.0f;
        z += pr[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
#pragma unroll
      for (int i = 0; i < VPL; ++i) pr[i] = pr[i] / z;
      v = slot ? expf(xj - m) / z : 0.0f;
    } else {
      m = xj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
      const float ex = slot ? expf(xj - m) : 0.0f;
      z = ex;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
      v = slot ? ex / z : 0.0f;
    }
    // renormalisation and scale
    float gv;
    if (renorm) {
      float S = v, dot = gw * v;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        S += __shfl_xor_sync(FULL, S, off);
        dot += __shfl_xor_sync(FULL, dot, off);
      }
      gv = slot ? scale / S * (gw - dot / S) : 0.0f;
    } else {
      gv = slot ? scale * gw : 0.0f;
    }
    float D = v * gv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) D += __shfl_xor_sync(FULL, D, off);
    // the row in two stores: every element as if unselected (softmax before
    // top-k: p * (0 - D); otherwise 0) by its owner lane, 16 bytes at a time,
    // then after __syncwarp (which orders the warp's memory operations) each
    // slot lane overwrites its selected expert (the selected experts of a
    // token are distinct)
    const bool prerow = score_fn != MOE_SIGMOID && pre;
    float* grow = grad_logits + t * E;
    float val[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) val[i] = prerow ? pr[i] * (0.0f - D) : 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int ee = lane * VPL + i;
      if (vec) {
        if ((i & 3) == 0 && i + 3 < VPL)
          __stcs(reinterpret_cast<float4*>(grow + ee), make_float4(val[i], val[i + 1], val[i + 2], val[i + 3]));
      } else if (ee < E) {
        __stcs(grow + ee, val[i]);
      }
    }
    __syncwarp();
    if (slot) {
      float gs;
      if (score_fn == MOE_SIGMOID) gs = gv * v * (1.0f - v);
      else gs = v * (gv - D);  // softmax before top-k: p_e * (gp_e - D) with p_e = v; after: v * (gv - D)
      grow[e] = gs;
    }
  }
}

extern "C" int moe_aux_workspace_bytes(int32_t num_tokens, int32_t num_experts, size_t* bytes) {
  if (num_tokens < 0 || num_experts <= 0 || !bytes) return MOE_ERR_INVALID_ARG;
  if (num_experts > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  *bytes = aux_ws_bytes(num_experts);
  return MOE_OK;
}

// Test hook: div_rn_by_recip(a[i], b[i], 1/b[i]) against the IEEE quotient
// a[i] / b[i], bit for bit, for pairs inside the method's range; counts the
// mismatches into *mismatches (device, zeroed by the caller).
static __global__ void div_check_kernel(const float* __restrict__ a, const float* __restrict__ b, long long n,
                                 unsigned int* mismatches) {
  unsigned int bad = 0;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float x = a[i], d = b[i];
    if (!(x >= kDivMinNum && d >= kDivMinDen && d <= kDivMaxDen)) continue;
    const float y = 1.0f / d;
    bad += __float_as_uint(div_rn_by_recip(x, d, y)) != __float_as_uint(x / d);
  }
  if (bad) atomicAdd(mismatches, bad);
}

extern "C" int moe_debug_div_check(const float* a, const float* b, int64_t n, uint32_t* mismatches, void* stream) {
  if (n < 0 || (n > 0 && (!a || !b || !mismatches))) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
  div_check_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a, b, (long long)n,
                                                                            reinterpret_cast<unsigned int*>(mismatches));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_aux_scores(int32_t T, int32_t E, int32_t k, int32_t score_fn, const float* logits, float* probs,
                              uint8_t* routing_map, int32_t* tokens_per_expert, void* ws, size_t ws_bytes,
                              void* stream) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (score_fn != MOE_SOFTMAX && score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!tokens_per_expert || (T > 0 && (!logits || !probs || !routing_map))) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < aux_ws_bytes(E)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool aligned = ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(probs) |
                         reinterpret_cast<uintptr_t>(routing_map)) & 15) == 0;
  if (aligned && k <= 8 && (E == 64 || E == 128 || E == 256)) {
    // four tokens per warp; enough warps for every SM, each taking a few quads
    const long long nq = ((long long)T + 3) / 4;
    const int per_sm = E == 256 ? 2 : 3;  // resident blocks (the kernel's launch bounds; 3 measured faster than 4)
    const int grid = (int)std::max(1LL, std::min<long long>((nq + kQuadThreads / 32 - 1) / (kQuadThreads / 32),
                                                            (long long)sm_count() * per_sm));
    const size_t smem = (size_t)E * sizeof(int) + (size_t)(kQuadThreads / 32) * 32 * 8;
    cudaError_t err = cudaSuccess;
    if (E == 64)
      err = launch_pdl(aux_scores_quad_kernel<8>, dim3(grid), dim3(kQuadThreads), smem, st, T, k, score_fn, logits,
                       probs, routing_map, tokens_per_expert, ws);
    else if (E == 128)
      err = launch_pdl(aux_scores_quad_kernel<16>, dim3(grid), dim3(kQuadThreads), smem, st, T, k, score_fn, logits,
                       probs, routing_map, tokens_per_expert, ws);
    else
      err = launch_pdl(aux_scores_quad_kernel<32>, dim3(grid), dim3(kQuadThreads), smem, st, T, k, score_fn, logits,
                       probs, routing_map, tokens_per_expert, ws);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const int vpl = pick_vpl(E);
  const int grid = std::max(1, std::min((T + 15) / 16, sm_count() * 3));  // 3 blocks per SM (40 registers)
  // histogram, then 32 packed candidate keys per warp
  const size_t smem = (size_t)((E + 1) & ~1) * sizeof(int) + (size_t)(kScoreThreads / 32) * 32 * 8;
  cudaError_t err = cudaSuccess;
  MOE_VPL_SWITCH(vpl, (err = launch_pdl(aux_scores_kernel<V>, dim3(grid), dim3(kScoreThreads), smem, st, T, E, k,
                                        score_fn, logits, probs, routing_map, tokens_per_expert, ws)));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_aux_loss_fwd(int32_t T_rows, int32_t T_total, int32_t E, int32_t k, float coeff,
                                const float* probs, const int32_t* tokens_per_expert, float* loss, void* ws,
                                size_t ws_bytes, void* stream) {
  if (T_rows < 0 || T_total <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!loss || !tokens_per_expert || (T_rows > 0 && !probs)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < aux_ws_bytes(E)) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(probs) & 15) return MOE_ERR_INVALID_ARG;
  const double C = (double)coeff * (double)E / ((double)T_total * (double)k);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t err = launch_pdl(aux_loss_fwd_kernel, dim3(kLossBlocks), dim3(kLossThreads),
                                     (size_t)E * sizeof(float), st, (long long)T_rows * E, E, C, probs,
                                     tokens_per_expert, loss, ws);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_aux_scores_bwd(int32_t T, int32_t E, int32_t score_fn, const float* probs,
                                  const float* grad_probs, float* grad_logits, void* stream) {
  if (T < 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if (score_fn != MOE_SOFTMAX && score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (score_fn != MOE_SOFTMAX || E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!probs || !grad_probs || !grad_logits) return MOE_ERR_INVALID_ARG;
  const int vpl = pick_vpl(E);
  const int grid = std::max(1, std::min((T + kAuxWarps - 1) / kAuxWarps, sm_count() * 8));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  const bool aligned = ((reinterpret_cast<uintptr_t>(probs) | reinterpret_cast<uintptr_t>(grad_probs) |
                         reinterpret_cast<uintptr_t>(grad_logits)) & 15) == 0;
  MOE_VPL_SWITCH(vpl, (err = launch_pdl(aux_scores_bwd_kernel<V>, dim3(grid), dim3(kAuxThreads), 0, st, T, E, probs,
                                        grad_probs, grad_logits, aligned)));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_aux_scores_bwd_logits(int32_t T, int32_t E, int32_t score_fn, const float* logits,
                                         const float* grad_probs, float* grad_logits, void* stream) {
  if (T < 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if (score_fn != MOE_SOFTMAX && score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !grad_probs || !grad_logits) return MOE_ERR_INVALID_ARG;
  const int vpl = pick_vpl(E);
  const int grid = std::max(1, std::min((T + kAuxWarps - 1) / kAuxWarps, sm_count() * 8));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool aligned = ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(grad_probs) |
                         reinterpret_cast<uintptr_t>(grad_logits)) & 15) == 0;
  cudaError_t err = cudaSuccess;
  MOE_VPL_SWITCH(vpl, (err = launch_pdl(aux_scores_bwd_logits_kernel<V>, dim3(grid), dim3(kAuxThreads), 0, st, T,
                                        E, score_fn, logits, grad_probs, grad_logits, aligned)));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// blocks of route_weights_bwd_kernel<V> resident per SM (queried once per V)
template <int V>
int rw_resident_blocks() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, route_weights_bwd_kernel<V>, kAuxThreads, 0) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
  });
  return n;
}

extern "C" int moe_route_weights_bwd(const moe_route_params* p, const void* logits, const int32_t* topk_ids,
                                     const float* grad_weights, float* grad_logits, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (!p) return MOE_ERR_INVALID_ARG;
  const int T = p->num_tokens, E = p->num_experts, k = p->top_k;
  if (T < 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (p->score_fn != MOE_SOFTMAX && p->score_fn != MOE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (p->logits_dtype != MOE_F32 && p->logits_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS || k > 32) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_ids || !grad_weights || !grad_logits) return MOE_ERR_INVALID_ARG;
  if (ws && ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  const int vpl = pick_vpl(E);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  // one resident wave (the rows are grid-strided)
  MOE_VPL_SWITCH(vpl, (err = launch_pdl(route_weights_bwd_kernel<V>,
                                        dim3(std::max(1, std::min((T + kAuxWarps - 1) / kAuxWarps,
                                                                  sm_count() * rw_resident_blocks<V>()))),
                                        dim3(kAuxThreads), 0, st, T, E, k,
                                        p->score_fn, p->softmax_before_topk ? 1 : 0, p->renormalize ? 1 : 0,
                                        p->scaling_factor, logits, p->logits_dtype, topk_ids, grad_weights,
                                        grad_logits, reinterpret_cast<WsHeader*>(ws))));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_aux_loss_bwd(int32_t T_rows, int32_t T_total, int32_t E, int32_t k, float coeff,
                                const float* grad_loss, const float* probs, const int32_t* tokens_per_expert,
                                float* grad_probs, float* grad_logits, void* stream) {
  if (T_rows < 0 || T_total <= 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (!grad_loss || !tokens_per_expert || (T_rows > 0 && !probs)) return MOE_ERR_INVALID_ARG;
  if (T_rows == 0 || (!grad_probs && !grad_logits)) return MOE_OK;
  const float C = (float)((double)coeff * (double)E / ((double)T_total * (double)k));
  const int vpl = pick_vpl(E);
  const int grid = std::max(1, std::min((T_rows + kAuxWarps - 1) / kAuxWarps, sm_count() * 8));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = (size_t)E * sizeof(float);
  cudaError_t err = cudaSuccess;
  MOE_VPL_SWITCH(vpl, (err = launch_pdl(aux_loss_bwd_kernel<V>, dim3(grid), dim3(kAuxThreads), smem, st, T_rows, E,
                                        C, grad_loss, probs, tokens_per_expert, grad_probs, grad_logits)));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
