// moe_rmsnorm_router_topk: fused RMSNorm + router projection + top-k for small
// decode batches, with the projection on the 5th-generation tensor cores.
//
// Source: RMSNorm Router Top-K A2AV Kernel API Reference -- Background (fused
// RMSNorm and router top-K for T = B*S <= 128, producing normalised hidden
// states, top-K indices and masked affinities), Parameters (hidden_states,
// gamma, router_weights [H,E], router_bias, eps, top_k, router_act_fn),
// Returns, Notes (T <= 128; H % 128 == 0; ACT2: top-K on raw logits, then the
// activation on the selected experts only).
//
// Three launches chained by programmatic dependent launch: each kernel lets
// the next one be scheduled at its entry, and the next one does everything
// that does not read its predecessor's output (the router weights, gamma,
// barriers, TMEM) before waiting on it.
//
//   K1 rmsnorm_kernel, a block per token: the sum of exact squares of the row
//   in double, r_t = 1/sqrt(mean + eps) in double (kept as r_hi + r_lo in
//   fp32), then each x*gamma*r rounded once to bf16: x*gamma is exact in fp32,
//   its product with r_hi is rounded to fp32 and then to bf16; where that fp32
//   value is a bf16 rounding midpoint or one fp32 ulp from one, the side is
//   taken from the remainder (x*gamma*r_hi - p + x*gamma*r_lo, two fused
//   multiply-adds), so the bf16 value is the single rounding of x*gamma*r.
//   The result is out_norm.
//
//   K2 project_kernel, one CTA per (token group, expert group of 64, K-slice):
//   the slice's W chunks (64 rows x 64 experts) staged by 2-D TMA before the
//   wait, its out_norm chunks (tokens x 64 columns) after it, both with the
//   128-byte swizzle (the canonical K-major A / MN-major B layouts of
//   tcgen05.mma); one thread issues each chunk's M=128 x N=64 x K=16 MMAs into
//   TMEM as it lands; the fp32 partial logits go from TMEM to the workspace.
//   The token group size and the K-split KS are chosen so that every CTA is
//   resident at once with the fewest post-wait staged bytes per CTA plus
//   partial-logit bytes K3 reads per token (T=128, H=7168, E=256: two 64-token
//   groups x 4 expert groups x 16 slices of 7 chunks = 128 CTAs).
//
//   K3 select_kernel, a block per token: the logit of expert e is the sum of
//   its KS partials in slice order (fp32), then the bias, the top-k on the raw
//   logits (ties -> lower expert), ids and the masked bf16 affinities.
//
// No kernel waits on another's blocks: no grid-wide barrier, no cluster, no
// cooperative launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kProjThreads = 256;  // 8 warps: 4 TMEM lane quarters x 2 column halves
constexpr int kChunk = 64;         // hidden columns per staged chunk (one 128-byte swizzle atom)
constexpr int kExpGroup = 64;      // experts per CTA (MMA N <= 64)
constexpr int kM = 128;            // MMA M: token rows (a 64-token group pads with zero rows)
constexpr int kMaxE = 1024;        // top-k stage: 8 experts per lane per round of 256
constexpr int kMaxStages = 8;      // staged chunks in flight
constexpr int kMaxKS = 48;         // K-slices (bounds the partial-logit workspace)
constexpr int kATile = kM * 128;      // 16 KB
constexpr int kBTile = kChunk * 128;  // 8 KB (64 K rows x 64 experts)
constexpr int kSmemLimit = 227 * 1024;  // opt-in shared memory per CTA
constexpr int kSelThreads = 256;        // K3: threads summing the partial logits
constexpr int kMaxH = 32768;            // hidden size limit

struct DecodeArgs {
  const uint16_t* x;      // [T,H] bf16
  const uint16_t* gamma;  // [H]
  const uint16_t* bias;   // [E] or null
  uint16_t* out_norm;     // [T,H]
  int32_t* ids;           // [T,k]
  uint16_t* aff;          // [T,E]
  float* dbg_logits;      // [T,E] or null
  WsHeader* hdr;
  float* part;            // [KS][TG*TGS][NG*64] fp32 partial logits (workspace)
  int T, H, E, k, act;
  int KS;                 // K-slices
  int TGS;                // tokens per group: 64 or 128
  int TG;                 // token groups
  int NG;                 // expert groups
  int nch;                // H / 64
  int S;                  // ring stages
  float eps;
  long long timeout_ns;
};

// K2 shared-memory layout (offsets from a 1024-byte aligned base)
struct DecLayout {
  int a, b, bars, slot, flag, total;
};
__host__ __device__ inline DecLayout dec_layout(int S) {
  DecLayout L;
  L.a = 0;
  L.b = L.a + S * kATile;
  L.bars = L.b + S * kBTile;
  L.slot = L.bars + (2 * kMaxStages + 1) * 8;
  L.flag = L.slot + 16;
  L.total = L.flag + 16;
  return L;
}

// ---- tcgen05 helpers (inline PTX, sm_100a) ----
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(smem_dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor (tcgen05): start, leading/stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: D fp32, A/B bf16, A K-major, B MN-major, M=128, N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

// packed fp32 pairs (two IEEE round-to-nearest products per instruction)
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return (unsigned long long)__float_as_uint(lo) | ((unsigned long long)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long x, unsigned long long y) {
  unsigned long long z;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  return z;
}

// bf16 of x*gamma*r with one rounding, for 8 bf16 of x (a 16-byte group) and
// the matching gamma (as fp32); xg = x*gamma is exact in fp32 and r = rh + rl.
// p = fl32(xg*rh) is within one fp32 ulp of xg*r (half an ulp from rounding,
// at most half from dropping xg*rl), so it rounds to bf16 like the exact
// product unless p is a bf16 midpoint m or one ulp from it (low 16 bits
// 0x7fff, 0x8000 or 0x8001).  normalize8 reports whether that happened;
// normalize8_exact then takes the side of m from the sign of
// (p - m) + (xg*rh - p) + xg*rl (the middle term exact by a fused
// multiply-add) and nudges m one fp32 ulp that way before the bf16 rounding
// (an exact tie stays on m: round half to even).
__device__ __forceinline__ bool normalize8(uint4 xv, const unsigned long long* g2, float rh, uint4* out) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const unsigned long long r2 = pack2(rh, rh);
  uint32_t ow[4];
  uint32_t mid = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // (x*gamma)*rh for the two bf16 of the word: x*gamma exact, one rounding to fp32
    const unsigned long long p = mul2(mul2(pack2(__uint_as_float(xw[j] << 16), __uint_as_float(xw[j] & 0xffff0000u)), g2[j]), r2);
    const uint32_t u0 = (uint32_t)p, u1 = (uint32_t)(p >> 32);
    mid |= (uint32_t)((((u0 + 0x8001u) & 0xffffu) < 3u) | (((u1 + 0x8001u) & 0xffffu) < 3u));
    const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(u0), __uint_as_float(u1));
    ow[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *out = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  return mid != 0;
}

__device__ __noinline__ uint4 normalize8_exact(uint4 xv, const float* g, float rh, float rl) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  uint32_t ow[4];
  for (int j = 0; j < 8; ++j) {
    const float xg = __uint_as_float((j & 1) ? (xw[j >> 1] & 0xffff0000u) : (xw[j >> 1] << 16)) * g[j];
    const float p = xg * rh;
    uint32_t u = __float_as_uint(p);
    if (((u + 0x8001u) & 0xffffu) < 3u) {
      const uint32_t mb = (u & 0xffff0000u) | 0x8000u;  // the bf16 midpoint next to p
      const float m = __uint_as_float(mb);
      const float d = (p - m) + fmaf(xg, rl, fmaf(xg, rh, -p));  // p - m is exact
      u = mb;
      if (d != 0.0f) u += ((__float_as_uint(d) ^ mb) >> 31) ? 0xffffffffu : 1u;
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(u));
    const uint32_t hb = *reinterpret_cast<const uint16_t*>(&h);
    if (j & 1) ow[j >> 1] |= hb << 16;
    else ow[j >> 1] = hb;
  }
  return make_uint4(ow[0], ow[1], ow[2], ow[3]);
}

__device__ __forceinline__ double sumsq8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  double acc = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
    acc += (double)(lo * lo);  // squares of bf16 values are exact in fp32
    acc += (double)(hi * hi);
  }
  return acc;
}

// K3: ids, affinities (and debug logits) of one token from its logits row in
// shared memory; outputs are written only while the workspace status is
// MOE_OK.  R rounds of 256 experts: lane l holds experts r*256 + 8l .. +7 of
// round r in slots 8r .. 8r+7 (E is a multiple of 16, so a lane's 8 experts
// of a round are all present or all absent).
template <int R>
__device__ void select_row(const DecodeArgs& a, int t, int lane, const float* row, int status, const uint4* bv) {
  constexpr int NS = 8 * R;
  float lg[NS];
  uint32_t valid = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e0 = r * 256 + lane * 8;
    if (e0 < a.E) {
      const float4 u = reinterpret_cast<const float4*>(row + e0)[0];
      const float4 w = reinterpret_cast<const float4*>(row + e0)[1];
      lg[8 * r + 0] = u.x; lg[8 * r + 1] = u.y; lg[8 * r + 2] = u.z; lg[8 * r + 3] = u.w;
      lg[8 * r + 4] = w.x; lg[8 * r + 5] = w.y; lg[8 * r + 6] = w.z; lg[8 * r + 7] = w.w;
      valid |= 0xffu << (8 * r);
      if (a.bias) {
        const uint32_t bw[4] = {bv[r].x, bv[r].y, bv[r].z, bv[r].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          lg[8 * r + 2 * i] += __uint_as_float(bw[i] << 16);
          lg[8 * r + 2 * i + 1] += __uint_as_float(bw[i] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) lg[8 * r + i] = 0.0f;
    }
  }
  // top-k on the raw logits: k rounds of (warp max of the order-preserving
  // key, then the lowest expert holding it), ties -> lower expert
  uint32_t key[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) key[i] = ordered_key(lg[i]);
  uint32_t chosen = 0;
  int my_id = 0;
  if constexpr (R == 1) {
    // up to 256 experts: the lane's 8 keys sorted once, descending, by an
    // odd-even transposition network that swaps only on a strictly larger key
    // (stable: equal keys keep the lower slot, the lower expert, first;
    // absent slots carry key 0 and sink), so that each round pops the head in
    // one step instead of rescanning the lane
    uint32_t sk[8];
    int ss[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool v = (valid >> i) & 1u;
      sk[i] = v ? key[i] : 0u;
      ss[i] = v ? i : NS;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int i = r & 1; i + 1 < 8; i += 2)
        if (sk[i + 1] > sk[i]) {
          const uint32_t tk = sk[i];
          sk[i] = sk[i + 1];
          sk[i + 1] = tk;
          const int ts = ss[i];
          ss[i] = ss[i + 1];
          ss[i + 1] = ts;
        }
    for (int j = 0; j < a.k; ++j) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, sk[0]);
      const uint32_t win =
          __reduce_min_sync(0xffffffffu, (ss[0] < NS && sk[0] == m) ? (uint32_t)(lane * 8 + ss[0]) : 0xffffffffu);
      if (ss[0] < NS && (uint32_t)(lane * 8 + ss[0]) == win) {
        chosen |= 1u << ss[0];
#pragma unroll
        for (int i = 0; i < 7; ++i) {
          sk[i] = sk[i + 1];
          ss[i] = ss[i + 1];
        }
        sk[7] = 0u;
        ss[7] = NS;
      }
      if (lane == j) my_id = (int)win;
    }
  } else {
    uint32_t avail = valid;
    uint32_t bk = 0u;
    int bi = NS;  // this lane's best remaining (key, slot); slot NS = none
    auto lane_best = [&]() {
      bk = 0u;
      bi = NS;
#pragma unroll
      for (int i = NS - 1; i >= 0; --i)
        if (((avail >> i) & 1u) && key[i] >= bk) {  // from the top down: ties -> the lower slot (lower expert)
          bk = key[i];
          bi = i;
        }
    };
    auto slot_expert = [&](int i) { return (i >> 3) * 256 + lane * 8 + (i & 7); };
    lane_best();
    for (int j = 0; j < a.k; ++j) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t win =
          __reduce_min_sync(0xffffffffu, (bi < NS && bk == m) ? (uint32_t)slot_expert(bi) : 0xffffffffu);
      if (bi < NS && (uint32_t)slot_expert(bi) == win) {
        avail &= ~(1u << bi);
        chosen |= 1u << bi;
        lane_best();
      }
      if (lane == j) my_id = (int)win;
    }
  }
  if (status != MOE_OK) return;
  if (a.dbg_logits) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e0 = r * 256 + lane * 8;
      if (e0 < a.E) {
        float* d = a.dbg_logits + (size_t)t * a.E + e0;
        *reinterpret_cast<float4*>(d) = make_float4(lg[8 * r], lg[8 * r + 1], lg[8 * r + 2], lg[8 * r + 3]);
        *reinterpret_cast<float4*>(d + 4) = make_float4(lg[8 * r + 4], lg[8 * r + 5], lg[8 * r + 6], lg[8 * r + 7]);
      }
    }
  }
  // activation over the selected only (ACT2): sigmoid each, or softmax over the k
  float m = -INFINITY, ssum = 0.0f;
  if (a.act == MOE_SOFTMAX) {
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if ((chosen >> i) & 1u) m = fmaxf(m, lg[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if ((chosen >> i) & 1u) ssum += expf(lg[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
  }
  if (lane < a.k) a.ids[(size_t)t * a.k + lane] = my_id;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e0 = r * 256 + lane * 8;
    if (e0 >= a.E) continue;
    uint32_t ow[4];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int s0 = 8 * r + i;
      float v0 = 0.0f, v1 = 0.0f;
      if ((chosen >> s0) & 1u) v0 = (a.act == MOE_SOFTMAX) ? expf(lg[s0] - m) / ssum : sigmoid_f32(lg[s0]);
      if ((chosen >> (s0 + 1)) & 1u)
        v1 = (a.act == MOE_SOFTMAX) ? expf(lg[s0 + 1] - m) / ssum : sigmoid_f32(lg[s0 + 1]);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
      ow[i / 2] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&h0)) |
                  ((uint32_t)(*reinterpret_cast<const uint16_t*>(&h1)) << 16);
    }
    *reinterpret_cast<uint4*>(a.aff + (size_t)t * a.E + e0) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

// K1: RMSNorm, a block per token row.  Sum of exact squares in double (a fixed
// order: thread partials, a shuffle tree, warps in order), r = 1/sqrt(mean +
// eps) in double kept as r_hi + r_lo, then x*gamma*r rounded once to bf16
// (normalize8 / normalize8_exact) into out_norm.  gamma is read before the
// dependency wait (a weight, not written by the preceding kernel).
constexpr int kNormThreads = 512;
constexpr int kNormKeep = 2;  // 16-byte groups a thread keeps in registers (H <= 8192)

__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const DecodeArgs a) {
  __shared__ double red[kNormThreads / 32];
  __shared__ float2 rr;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nq = a.H / 8;  // 16-byte groups in a row
  uint4 gkeep[kNormKeep];
#pragma unroll
  for (int j = 0; j < kNormKeep; ++j) {
    const int qq = tid + j * kNormThreads;
    gkeep[j] = qq < nq ? __ldg(reinterpret_cast<const uint4*>(a.gamma) + qq) : make_uint4(0, 0, 0, 0);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the hidden states are the preceding kernel's output
  const uint16_t* xr = a.x + (size_t)t * a.H;
  uint4 keep[kNormKeep];
  double acc = 0.0;
#pragma unroll
  for (int j = 0; j < kNormKeep; ++j) {
    const int qq = tid + j * kNormThreads;
    keep[j] = qq < nq ? __ldcg(reinterpret_cast<const uint4*>(xr) + qq) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int j = 0; j < kNormKeep; ++j) acc += sumsq8(keep[j]);
  for (int qq = tid + kNormKeep * kNormThreads; qq < nq; qq += kNormThreads)
    acc += sumsq8(__ldcg(reinterpret_cast<const uint4*>(xr) + qq));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  if (tid == 0) {
    double ss = 0.0;
    for (int w = 0; w < kNormThreads / 32; ++w) ss += red[w];
    const double r = 1.0 / sqrt(ss / (double)a.H + (double)a.eps);
    const float rh = (float)r;
    rr = make_float2(rh, (float)(r - (double)rh));
  }
  __syncthreads();
  const float2 r2 = rr;
  uint16_t* orow = a.out_norm + (size_t)t * a.H;
  auto normalise = [&](int qq, uint4 xv, uint4 gv) {
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
    float g[8];
    unsigned long long g2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      g[2 * i] = __uint_as_float(gw[i] << 16);
      g[2 * i + 1] = __uint_as_float(gw[i] & 0xffff0000u);
      g2[i] = pack2(g[2 * i], g[2 * i + 1]);
    }
    uint4 o;
    if (normalize8(xv, g2, r2.x, &o)) o = normalize8_exact(xv, g, r2.x, r2.y);  // a bf16 midpoint (rare)
    reinterpret_cast<uint4*>(orow)[qq] = o;
  };
#pragma unroll
  for (int j = 0; j < kNormKeep; ++j)
    if (tid + j * kNormThreads < nq) normalise(tid + j * kNormThreads, keep[j], gkeep[j]);
  for (int qq = tid + kNormKeep * kNormThreads; qq < nq; qq += kNormThreads)
    normalise(qq, __ldcg(reinterpret_cast<const uint4*>(xr) + qq), __ldg(reinterpret_cast<const uint4*>(a.gamma) + qq));
}

// K2: the partial logits of one (token group, expert group, K-slice).
__global__ void __launch_bounds__(kProjThreads, 1)
    project_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // 1024-byte aligned (swizzle atoms)
  const int TGS = a.TGS, S = a.S;
  const DecLayout L = dec_layout(S);
  uint8_t* sA = smem + L.a;
  uint8_t* sB = smem + L.b;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);  // both copies of the stage landed
  uint64_t* empty = full + kMaxStages;                          // the stage's MMAs are done
  uint64_t* mma_bar = empty + kMaxStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.slot);
  volatile int* flag = reinterpret_cast<volatile int*>(smem + L.flag);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int ks = blockIdx.x % a.KS, rest = blockIdx.x / a.KS;
  const int ng = rest % a.NG, tg = rest / a.NG;
  const int row0 = tg * TGS;               // first token of the group
  const int e0 = ng * kExpGroup;           // first expert of the group
  const int N = min(kExpGroup, a.E - e0);  // multiple of 16
  const int c0 = (int)((long long)a.nch * ks / a.KS);
  const int nb = (int)((long long)a.nch * (ks + 1) / a.KS) - c0;  // chunks of this CTA (>= 1)
  const int nres = min(S, nb);
  const uint32_t stage_tx = (uint32_t)(TGS * 128 + kBTile);

  int issued = 0;  // chunks whose copies have been issued (thread 0)
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(mma_bar, 1);
    flag[0] = 0;
    // before the dependency wait, only the router weights (not written by the
    // preceding kernel); each stage's barrier expects both of its copies
    for (int s = 0; s < nres; ++s) {
      mbar_arrive_expect_tx(full + s, stage_tx);
      tma_load_2d(sB + s * kBTile, &wmap, e0, (c0 + s) * kChunk, full + s);
    }
  }
  if (warp == 0) tmem_alloc(tmem_slot, 64);
  // with 64-token groups, A rows 64..127 are zero in every stage (the TMA box fills rows 0..63)
  if (TGS < kM)
    for (int i = tid; i < S * ((kM - TGS) * 8); i += kProjThreads) {
      const int s = i / ((kM - TGS) * 8), off = i % ((kM - TGS) * 8);
      *reinterpret_cast<uint4*>(sA + s * kATile + TGS * 128 + off * 16) = make_uint4(0, 0, 0, 0);
    }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // the normalised rows are K1's output
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    for (; issued < nres; ++issued)
      tma_load_2d(sA + issued * kATile, &xmap, (c0 + issued) * kChunk, row0, full + issued);
    // ---------------- project: each chunk's MMAs as soon as it has landed ----------------
    const uint32_t idesc = idesc_bf16_f32(N);
    bool mma_issued = false;
    for (int i = 0; i < nb; ++i) {
      const int s = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      if (!mbar_wait_bounded(full + s, ph, a.timeout_ns)) {
        record_timeout(a.hdr);
        flag[0] = 1;
        break;
      }
      tc_fence_after();
      const uint32_t aBase = smem_addr(sA + s * kATile), bBase = smem_addr(sB + s * kBTile);
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk) {
        const uint64_t ad = smem_desc_sw128(aBase + kk * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(bBase + kk * 2048, 8192, 1024);
        umma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(empty + s);
      mma_issued = true;
      if (issued < nb) {
        // refill this stage with chunk i + S once its MMAs have read it
        if (!mbar_wait_bounded(empty + s, ph, a.timeout_ns)) {
          record_timeout(a.hdr);
          flag[0] = 1;
          break;
        }
        mbar_arrive_expect_tx(full + s, stage_tx);
        tma_load_2d(sA + s * kATile, &xmap, (c0 + issued) * kChunk, row0, full + s);
        tma_load_2d(sB + s * kBTile, &wmap, e0, (c0 + issued) * kChunk, full + s);
        ++issued;
      }
    }
    // one commit tracks every MMA this thread issued: its arrival means they
    // have all finished reading shared memory and writing TMEM
    bool drained = !mma_issued;
    if (mma_issued) {
      umma_commit(mma_bar);
      drained = mbar_wait_bounded(mma_bar, 0, a.timeout_ns);
      if (!drained) {
        record_timeout(a.hdr);
        flag[0] = 1;
      }
    }
    if (flag[0]) {
      // a wait gave up: let the MMAs (if their commit has not arrived yet, wait
      // once more, bounded) and the copies still in flight finish before the
      // CTA frees its TMEM and exits
      if (!drained) mbar_wait_bounded(mma_bar, 0, a.timeout_ns);
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_bounded(full + (i % S), (uint32_t)(i / S) & 1u, a.timeout_ns);
    }
  }
  __syncthreads();
  // ---------------- partial logits: TMEM -> the workspace ----------------
  // warp w reads TMEM lanes 32*(w%4).. (token rows) and column half w/4; each
  // thread stores its row's 32 fp32 (128 contiguous bytes)
  if (flag[0] == 0) {
    const int wq = warp & 3, ch = warp >> 2;
    if (wq * 32 < TGS && ch * 32 < N) {
      tc_fence_after();
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(ch * 32), v);
      const int row = wq * 32 + lane;
      float4* d = reinterpret_cast<float4*>(a.part + ((size_t)ks * (a.TG * TGS) + row0 + row) * (a.NG * kExpGroup) + e0 + ch * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// K3: the logits of one token (its partials summed in slice order) and its top-k.
template <int R>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const DecodeArgs a) {
  __shared__ __align__(16) float row[kMaxE];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int t = blockIdx.x;
  uint4 bv[R];  // the bias of lane l's experts r*256 + 8l .. +7 (warp 0), a weight
#pragma unroll
  for (int r = 0; r < R; ++r) {
    bv[r] = make_uint4(0, 0, 0, 0);
    const int e0 = r * 256 + threadIdx.x * 8;
    if (threadIdx.x < 32 && a.bias && e0 < a.E) bv[r] = __ldg(reinterpret_cast<const uint4*>(a.bias + e0));
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partial logits are K2's output
  int status = MOE_OK;
  if (threadIdx.x < 32) status = *reinterpret_cast<const volatile int32_t*>(&a.hdr->status);
  const int tp = a.TG * a.TGS, ep = a.NG * kExpGroup;
  for (int e = threadIdx.x; e < a.E; e += kSelThreads) {
    const float* p = a.part + (size_t)t * ep + e;
    float sum = 0.0f;  // slice order
    if constexpr (R == 1) {
      // up to 256 experts: 4 loads in flight per thread (measured faster here than 16)
#pragma unroll 4
      for (int s = 0; s < a.KS; ++s) sum += __ldcg(p + (size_t)s * tp * ep);
    } else {
      // more experts: 16 slices' loads in flight at a time (one L2 round trip for KS <= 16)
      for (int s0 = 0; s0 < a.KS; s0 += 16) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = s0 + j < a.KS ? __ldcg(p + (size_t)(s0 + j) * tp * ep) : 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (s0 + j < a.KS) sum += v[j];
      }
    }
    row[e] = sum;
  }
  __syncthreads();
  if (threadIdx.x < 32) select_row<R>(a, t, threadIdx.x, row, status, bv);
}

// ---- host ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr int kDecSmemMax = kSmemLimit;

// Per device: the kernel attribute set once, and the SM count.
struct DecDevice {
  std::once_flag once;
  int ok = 0;
  int sms = 0;
};
DecDevice g_dec_dev[64];

int dec_device_setup(int dev) {
  DecDevice& d = g_dec_dev[dev];
  std::call_once(d.once, [&d, dev] {
    if (cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemMax) !=
        cudaSuccess)
      return;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || d.sms < 1) return;
    d.ok = 1;
  });
  return d.ok;
}

struct DecPlan {
  int KS, NG, TG, TGS, nch, S, smem;
};

// Choose the token group size and the K-split: every CTA resident at once
// (one per SM), least cost = post-wait staged bytes per CTA (the normalised
// rows) + the partial logits K3 reads per token.
DecPlan dec_plan(int T, int H, int E, int sms) {
  DecPlan best = {};
  double best_cost = 1e300;
  const int nch = H / kChunk;
  const int NG = (E + kExpGroup - 1) / kExpGroup;
  for (int tgs = 64; tgs <= 128; tgs += 64) {
    if (tgs == 128 && T <= 64) continue;
    const int TG = (T + tgs - 1) / tgs;
    for (int ks = 1; ks <= std::min(nch, kMaxKS); ++ks) {
      if (TG * NG * ks > sms && ks > 1) break;
      DecPlan p;
      p.KS = ks;
      p.NG = NG;
      p.TG = TG;
      p.TGS = tgs;
      p.nch = nch;
      const int maxb = (nch + ks - 1) / ks;
      p.S = std::min(kMaxStages, maxb);
      p.smem = 1024 + dec_layout(p.S).total;
      // post-wait staged bytes per CTA (a ring stages the rows a second
      // time) + the partial logits K3 reads per token
      const double cost = (double)maxb * tgs * 128 * (maxb > p.S ? 2.0 : 1.0) + (double)ks * NG * kExpGroup * 4;
      if (cost < best_cost) {
        best_cost = cost;
        best = p;
      }
    }
  }
  return best;
}

size_t dec_ws_bytes(int T, int H, int E) {
  const int NG = (E + kExpGroup - 1) / kExpGroup;
  const int tp = T <= 64 ? 64 : 128;
  return sizeof(WsHeader) + (size_t)std::min(H / kChunk, kMaxKS) * tp * NG * kExpGroup * sizeof(float);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_rmsnorm_router_topk_workspace_bytes(int32_t T, int32_t H, int32_t E, size_t* bytes) {
  if (T < 0 || T > 128 || H <= 0 || H % 128 != 0 || E <= 0 || !bytes) return MOE_ERR_INVALID_ARG;
  if (E % 16 != 0 || E > kMaxE || H > kMaxH) return MOE_ERR_UNSUPPORTED;
  *bytes = dec_ws_bytes(T, H, E);
  return MOE_OK;
}

extern "C" int moe_rmsnorm_router_topk(int32_t T, int32_t H, int32_t E, int32_t k, float eps, int32_t act,
                                       const void* hidden, const void* gamma, const void* W, const void* bias,
                                       void* out_norm, int32_t* ids, void* affinities, float* debug_logits, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (T < 0 || T > 128 || H <= 0 || H % 128 != 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (act != MOE_SIGMOID && act != MOE_SOFTMAX) return MOE_ERR_INVALID_ARG;
  if (E % 16 != 0 || E > kMaxE || k > MOE_MAX_TOPK || H > kMaxH) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!hidden || !gamma || !W || !out_norm || !ids || !affinities) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(gamma) | reinterpret_cast<uintptr_t>(W) |
       reinterpret_cast<uintptr_t>(out_norm) | reinterpret_cast<uintptr_t>(affinities) |
       reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(debug_logits)) & 15)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < dec_ws_bytes(T, H, E) || (reinterpret_cast<uintptr_t>(ws) & 15)) return MOE_ERR_WORKSPACE;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return MOE_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (!dec_device_setup(dev)) return MOE_ERR_CUDA;
  const DecPlan plan = dec_plan(T, H, E, g_dec_dev[dev].sms);
  if (plan.KS < 1) return MOE_ERR_UNSUPPORTED;

  DecodeArgs a = {};
  a.x = reinterpret_cast<const uint16_t*>(hidden);
  a.gamma = reinterpret_cast<const uint16_t*>(gamma);
  a.bias = reinterpret_cast<const uint16_t*>(bias);
  a.out_norm = reinterpret_cast<uint16_t*>(out_norm);
  a.ids = ids;
  a.aff = reinterpret_cast<uint16_t*>(affinities);
  a.dbg_logits = debug_logits;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  a.part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + sizeof(WsHeader));
  a.T = T;
  a.H = H;
  a.E = E;
  a.k = k;
  a.act = act;
  a.KS = plan.KS;
  a.TGS = plan.TGS;
  a.TG = plan.TG;
  a.NG = plan.NG;
  a.nch = plan.nch;
  a.S = plan.S;
  a.eps = eps;
  a.timeout_ns = kDefaultTimeoutNs;

  // out_norm [T][H]: dim0 = H (contiguous), dim1 = T; 64 x TGS boxes (rows past T read as zero)
  // W [H][E]: dim0 = E (contiguous), dim1 = H; 64 x 64 boxes (experts past E read as zero)
  CUtensorMap xmap, wmap;
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t gstride[1] = {(cuuint64_t)H * 2};
    const cuuint32_t xbox[2] = {64, (cuuint32_t)plan.TGS};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out_norm, gdim, gstride, xbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MOE_ERR_INVALID_ARG;
  }
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)E, (cuuint64_t)H};
    const cuuint64_t gstride[1] = {(cuuint64_t)E * 2};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MOE_ERR_INVALID_ARG;
  }

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_pdl(rmsnorm_kernel, dim3(T), dim3(kNormThreads), 0, st, a) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_pdl(project_kernel, dim3(plan.KS * plan.NG * plan.TG), dim3(kProjThreads), (size_t)plan.smem, st, a,
                 xmap, wmap) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int R = (E + 255) / 256;
  const cudaError_t e3 = R == 1   ? launch_pdl(select_kernel<1>, dim3(T), dim3(kSelThreads), 0, st, a)
                         : R == 2 ? launch_pdl(select_kernel<2>, dim3(T), dim3(kSelThreads), 0, st, a)
                         : R == 3 ? launch_pdl(select_kernel<3>, dim3(T), dim3(kSelThreads), 0, st, a)
                                  : launch_pdl(select_kernel<4>, dim3(T), dim3(kSelThreads), 0, st, a);
  if (e3 != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
