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
// One cooperative launch over G blocks; block c owns K-slice(s) of 128 hidden
// columns and the matching 128 rows of W.
//   phase 1  W slice -> shared memory by 2-D TMA (128-byte swizzle, the
//            canonical MN-major operand layout of tcgen05.mma); 256 TMEM
//            columns allocated; per-token partial sum of squares of the slice
//            (double) -> workspace.  Bounded grid barrier.
//   phase 2  every block adds the partial sums in block order (deterministic)
//            and forms r_t = 1/sqrt(mean + eps) in double; normalises its
//            slice (x*gamma exact in fp32, times r_t in double, one rounding to
//            bf16), writes
//            out_norm and the same bf16 values to shared memory in the
//            K-major 128-byte-swizzled layout; one thread issues the
//            M=128 x N=E x K=16 tcgen05.mma steps into TMEM; the partial logits
//            go TMEM -> registers (tcgen05.ld) -> workspace.  Barrier.
//   phase 3  block c sums the G partial logits of its tokens in block order,
//            adds the bias, and writes ids (top-k on the raw logits, ties ->
//            lower expert) and the masked bf16 affinities.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kKC = 128;         // hidden columns (MMA K) per slice
constexpr int kM = 128;          // MMA M (tokens, zero-padded)
constexpr int kMaxE = 256;       // MMA N limit
constexpr int kSmemMin = 120 * 1024;  // > half an SM's shared memory: one block (and TMEM user) per SM

struct DecodeArgs {
  const uint16_t* x;      // [T,H] bf16
  const uint16_t* gamma;  // [H]
  const uint16_t* bias;   // [E] or null
  uint16_t* out_norm;     // [T,H]
  int32_t* ids;           // [T,k]
  uint16_t* aff;          // [T,E]
  float* dbg_logits;      // [T,E] or null
  WsHeader* hdr;
  double* sumsq;          // [G][kM]
  float* plogits;         // [G][kM][NP]
  int T, H, E, k, act;
  int NP;                 // E rounded up to 64 (B tile columns)
  int N;                  // MMA N = E rounded up to 16
  int G;
  int nslices;            // H / kKC
  float eps;
  long long timeout_ns;
};

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

// double -> bf16 bits, one rounding to nearest-even: truncate to fp32 and set
// the last bit if anything was cut (round to odd), then round to nearest-even
// at bf16 precision; with >= 2 extra bits this equals direct rounding (Boldo &
// Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
// using rounding to odd", IEEE Trans. Computers 2008).
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double y) {
  float f = __double2float_rz(y);
  if ((double)f != y) f = __uint_as_float(__float_as_uint(f) | 1u);
  const __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the swizzled operand tiles
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int NB = a.NP / 64;                         // 64-column N boxes
  uint8_t* sA = smem;                               // [2 K-blocks][128 rows][128 B]  = 32 KB
  uint8_t* sB = smem + 32 * 1024;                   // [2 K-blocks][NB][64 rows][128 B] = NB * 16 KB
  uint8_t* tail = sB + NB * 16 * 1024;
  uint64_t* tma_bar = reinterpret_cast<uint64_t*>(tail);
  uint64_t* mma_bar = tma_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 16);
  int* flag = reinterpret_cast<int*>(tail + 32);    // [0] barrier scratch, [1] failure
  double* r_s = reinterpret_cast<double*>(tail + 64); // [kM]

  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t gen = barrier_generation(a.hdr);
  const uint32_t ncols = a.N <= 32 ? 32u : (a.N <= 64 ? 64u : (a.N <= 128 ? 128u : 256u));
  const int sl0 = (int)((long long)a.nslices * c / a.G), sl1 = (int)((long long)a.nslices * (c + 1) / a.G);

  if (tid == 0) {
    mbar_init(tma_bar, 1);
    mbar_init(mma_bar, 1);
    flag[1] = 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, ncols);
  // zero the A rows of padding tokens once (they stay zero for every slice)
  for (int i = tid; i < (kM - a.T) * 2 * 8; i += kDecThreads) {
    const int r = a.T + i / 16, kb = (i / 8) & 1, q = i & 7;
    *reinterpret_cast<uint4*>(sA + kb * 16384 + r * 128 + q * 16) = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---------------- phase 1: partial sums of squares ----------------
  // two threads per token, 64 columns each per slice; squares of bf16 values
  // are exact, and are summed in double
  {
    const int t = tid >> 1, half = tid & 1;
    double acc = 0.0;
    if (t < a.T) {
      for (int sl = sl0; sl < sl1; ++sl) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H + sl * kKC + half * 64);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 q = __ldg(src + v);
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
            acc += (double)(lo * lo);
            acc += (double)(hi * hi);
          }
        }
      }
    }
    double d = acc;
    d += __shfl_xor_sync(0xffffffffu, d, 1);
    if (half == 0 && t < kM) a.sumsq[(size_t)c * kM + t] = d;
  }
  bool ok = grid_barrier(a.hdr, (uint32_t)a.G, gen, a.timeout_ns, flag);

  // ---------------- phase 2: normalise, project ----------------
  if (ok) {
    // warp w reduces tokens w, w+8, ...: lane l adds the partials of blocks
    // l, l+32, ... (all loads in flight), then a fixed shuffle tree; every
    // block computes the same r_t
    for (int t = warp; t < a.T; t += kDecWarps) {
      double sv[5];
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int cp = lane + 32 * i;
        sv[i] = cp < a.G ? __ldcg(&a.sumsq[(size_t)cp * kM + t]) : 0.0;
      }
      double s = (sv[0] + sv[1]) + (sv[2] + sv[3]) + sv[4];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) r_s[t] = 1.0 / sqrt(s / (double)a.H + (double)a.eps);
    }
    __syncthreads();
    const uint32_t idesc = idesc_bf16_f32(a.N);
    uint32_t phase = 0;
    for (int sl = sl0; sl < sl1 && ok; ++sl) {
      if (tid == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_expect_tx(tma_bar, (uint32_t)(NB * 16 * 1024));
        for (int kb = 0; kb < 2; ++kb)
          for (int nb = 0; nb < NB; ++nb)
            tma_load_2d(sB + (kb * NB + nb) * 8192, &wmap, nb * 64, sl * kKC + kb * 64, tma_bar);
      }
      // normalised slice: (token, 16-byte group) pairs, 16 groups per token row;
      // a thread's loads are all issued before any is used
      constexpr int kPer = (kM * 16) / kDecThreads;  // pairs per thread (8)
      uint4 xb[kPer];
      const uint4 gv = __ldg(reinterpret_cast<const uint4*>(a.gamma + sl * kKC + (tid & 15) * 8));
#pragma unroll
      for (int b = 0; b < kPer; ++b) {
        const int i = tid + b * kDecThreads;
        const int t = i >> 4, q = i & 15;
        xb[b] = t < a.T ? __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H + sl * kKC + q * 8))
                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int b = 0; b < kPer; ++b) {
        const int i = tid + b * kDecThreads;
        const int t = i >> 4, q = i & 15;
        if (t >= a.T) continue;
        const size_t off = (size_t)t * a.H + sl * kKC + q * 8;
        const uint4 xv = xb[b];
        const double r = r_s[t];
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, gw[4] = {gv.x, gv.y, gv.z, gv.w};
        uint32_t ow[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x0 = __uint_as_float(xw[j] << 16), x1 = __uint_as_float(xw[j] & 0xffff0000u);
          const float g0 = __uint_as_float(gw[j] << 16), g1 = __uint_as_float(gw[j] & 0xffff0000u);
          // x*gamma is exact in fp32; the product with r is formed in double and
          // rounded once to bf16
          ow[j] = (uint32_t)f64_to_bf16_bits((double)(x0 * g0) * r) |
                  ((uint32_t)f64_to_bf16_bits((double)(x1 * g1) * r) << 16);
        }
        const uint4 o = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        *reinterpret_cast<uint4*>(a.out_norm + off) = o;
        const int kb = q >> 3, cq = q & 7;
        *reinterpret_cast<uint4*>(sA + kb * 16384 + t * 128 + ((cq ^ (t & 7)) << 4)) = o;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (tid == 0) {
        if (!mbar_wait_bounded(tma_bar, phase, a.timeout_ns)) {
          record_timeout(a.hdr);
          flag[1] = 1;
        } else {
          tc_fence_after();
          const uint32_t aBase = smem_addr(sA), bBase = smem_addr(sB);
#pragma unroll
          for (int ks = 0; ks < kKC / 16; ++ks) {
            const int kb = ks >> 2, kk = ks & 3;
            const uint64_t ad = smem_desc_sw128(aBase + kb * 16384 + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(bBase + kb * NB * 8192 + kk * 2048, 8192, 1024);
            umma_bf16(tmem, ad, bd, idesc, (sl > sl0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(mma_bar);
        }
      }
      __syncthreads();
      if (flag[1]) {
        ok = false;
        break;
      }
      // the MMAs must finish before the operand tiles are rewritten (next slice) or read out
      if (!mbar_wait_bounded(mma_bar, phase, a.timeout_ns)) {
        record_timeout(a.hdr);
        flag[1] = 1;
      }
      phase ^= 1u;
      __syncthreads();
      if (flag[1]) ok = false;
    }
    if (ok) {
      tc_fence_after();
      // TMEM -> registers -> workspace: warp w reads lanes 32*(w%4).., columns half (w/4)
      const int lb = (warp & 3) * 32;
      const int t = lb + lane;
      const int chalf = a.N > 128 ? 128 : a.N;  // columns per warp half
      for (int c0 = (warp >> 2) * chalf; c0 < min(a.N, ((warp >> 2) + 1) * chalf); c0 += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)lb << 16) + (uint32_t)c0, v);
        if (t < a.T) {
          float* dst = a.plogits + ((size_t)c * kM + t) * a.NP + c0;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (c0 + i < a.NP) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ncols);
  if (!ok) {
    // let the other blocks pass the second barrier quickly; outputs are undefined
    grid_barrier(a.hdr, (uint32_t)a.G, gen + 1, a.timeout_ns, flag);
    return;
  }
  if (!grid_barrier(a.hdr, (uint32_t)a.G, gen + 1, a.timeout_ns, flag)) return;

  // ---------------- phase 3: reduce partial logits, top-k, affinities ----------------
  // For each token of this block, warp w adds the partial logits of blocks
  // w, w+8, ... (lane = 8 experts; all loads of a warp in flight), the 8 warp
  // sums meet in shared memory and warp 0 adds them in warp order.
  float* red = reinterpret_cast<float*>(sA);  // [kDecWarps][NP], the operand tiles are free now
  const int t0 = (int)((long long)a.T * c / a.G), t1 = (int)((long long)a.T * (c + 1) / a.G);
  for (int t = t0; t < t1; ++t) {
    {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
      if (lane * 8 < a.NP) {
        constexpr int kB = 8;
        for (int cp0 = warp; cp0 < a.G; cp0 += kDecWarps * kB) {
          float4 u[kB], w[kB];
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            const int cp = cp0 + b * kDecWarps;
            if (cp < a.G) {
              const float* src = a.plogits + ((size_t)cp * kM + t) * a.NP + lane * 8;
              u[b] = __ldcg(reinterpret_cast<const float4*>(src));
              w[b] = __ldcg(reinterpret_cast<const float4*>(src + 4));
            } else {
              u[b] = w[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
#pragma unroll
          for (int b = 0; b < kB; ++b) {
            acc[0] += u[b].x; acc[1] += u[b].y; acc[2] += u[b].z; acc[3] += u[b].w;
            acc[4] += w[b].x; acc[5] += w[b].y; acc[6] += w[b].z; acc[7] += w[b].w;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) red[warp * a.NP + lane * 8 + i] = acc[i];
      }
    }
    __syncthreads();
    if (warp != 0) {
      __syncthreads();
      continue;
    }
    float lg[8];
    float bsum[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lg[i] = 0.0f;
      const int e = lane * 8 + i;
      bsum[i] = (a.bias && e < a.E) ? bf16_bits_to_f32(a.bias[e]) : 0.0f;
    }
    if (lane * 8 < a.NP) {
      for (int w = 0; w < kDecWarps; ++w)
#pragma unroll
        for (int i = 0; i < 8; ++i) lg[i] += red[w * a.NP + lane * 8 + i];
    }
    uint32_t valid = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      lg[i] += bsum[i];
      if (e < a.E) valid |= 1u << i;
      if (a.dbg_logits && e < a.E) a.dbg_logits[(size_t)t * a.E + e] = lg[i];
    }
    // top-k on the raw logits: k rounds of warp argmax, ties -> lower expert
    uint32_t chosen = 0, avail = valid;
    int my_id = 0;
    for (int j = 0; j < a.k; ++j) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((avail >> i) & 1u) {
          const unsigned long long pk = pack_key(lg[i], lane * 8 + i);
          best = pk > best ? pk : best;
        }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long o = shfl_xor_u64(0xffffffffu, best, off);
        best = o > best ? o : best;
      }
      const int win = packed_expert(best);
      const int owner = win >> 3;
      if (lane == owner) {
        avail &= ~(1u << (win & 7));
        chosen |= 1u << (win & 7);
      }
      if (lane == j) my_id = win;
    }
    // activation over the selected only (ACT2): sigmoid each, or softmax over the k
    float m = -INFINITY, ssum = 0.0f;
    if (a.act == MOE_SOFTMAX) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((chosen >> i) & 1u) m = fmaxf(m, lg[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((chosen >> i) & 1u) ssum += expf(lg[i] - m);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, off);
    }
    if (lane < a.k) a.ids[(size_t)t * a.k + lane] = my_id;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < a.E) {
        float v = 0.0f;
        if ((chosen >> i) & 1u) v = (a.act == MOE_SOFTMAX) ? expf(lg[i] - m) / ssum : sigmoid_f32(lg[i]);
        const __nv_bfloat16 hb = __float2bfloat16_rn(v);
        a.aff[(size_t)t * a.E + e] = *reinterpret_cast<const uint16_t*>(&hb);
      }
    }
    __syncthreads();
  }
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

int dec_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

int dec_grid(int H) {
  const int ns = H / kKC;
  return std::max(1, std::min(ns, dec_sms()));
}

size_t dec_ws_bytes(int H, int E) {
  const int G = dec_grid(H);
  const int NP = (E + 63) / 64 * 64;
  return sizeof(WsHeader) + (size_t)G * kM * sizeof(double) + (size_t)G * kM * NP * sizeof(float);
}

int dec_smem(int E) {
  const int NB = (E + 63) / 64;
  const int need = 1024 + 32 * 1024 + NB * 16 * 1024 + 64 + kM * 8;
  return std::max(need, kSmemMin);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_rmsnorm_router_topk_workspace_bytes(int32_t T, int32_t H, int32_t E, size_t* bytes) {
  if (T < 0 || T > 128 || H <= 0 || H % 128 != 0 || E <= 0 || !bytes) return MOE_ERR_INVALID_ARG;
  if (E % 16 != 0 || E > kMaxE) return MOE_ERR_UNSUPPORTED;
  *bytes = dec_ws_bytes(H, E);
  return MOE_OK;
}

extern "C" int moe_rmsnorm_router_topk(int32_t T, int32_t H, int32_t E, int32_t k, float eps, int32_t act,
                                       const void* hidden, const void* gamma, const void* W, const void* bias,
                                       void* out_norm, int32_t* ids, void* affinities, float* debug_logits, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (T < 0 || T > 128 || H <= 0 || H % 128 != 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (act != MOE_SIGMOID && act != MOE_SOFTMAX) return MOE_ERR_INVALID_ARG;
  if (E % 16 != 0 || E > kMaxE || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!hidden || !gamma || !W || !out_norm || !ids || !affinities) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(gamma) | reinterpret_cast<uintptr_t>(W) |
       reinterpret_cast<uintptr_t>(out_norm)) & 15)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < dec_ws_bytes(H, E) || (reinterpret_cast<uintptr_t>(ws) & 15)) return MOE_ERR_WORKSPACE;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return MOE_ERR_CUDA;

  DecodeArgs a = {};
  a.x = reinterpret_cast<const uint16_t*>(hidden);
  a.gamma = reinterpret_cast<const uint16_t*>(gamma);
  a.bias = reinterpret_cast<const uint16_t*>(bias);
  a.out_norm = reinterpret_cast<uint16_t*>(out_norm);
  a.ids = ids;
  a.aff = reinterpret_cast<uint16_t*>(affinities);
  a.dbg_logits = debug_logits;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  a.G = dec_grid(H);
  a.sumsq = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(ws) + sizeof(WsHeader));
  a.plogits = reinterpret_cast<float*>(a.sumsq + (size_t)a.G * kM);
  a.T = T;
  a.H = H;
  a.E = E;
  a.k = k;
  a.act = act;
  a.NP = (E + 63) / 64 * 64;
  a.N = (E + 15) / 16 * 16;
  a.nslices = H / kKC;
  a.eps = eps;
  a.timeout_ns = kDefaultTimeoutNs;

  // W [H][E] bf16: dim0 = E (contiguous), dim1 = H; 64 x 64 boxes, 128-byte swizzle
  CUtensorMap wmap;
  const cuuint64_t gdim[2] = {(cuuint64_t)E, (cuuint64_t)H};
  const cuuint64_t gstride[1] = {(cuuint64_t)E * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return MOE_ERR_INVALID_ARG;

  const int smem = dec_smem(E);
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.G);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel, a, wmap);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
