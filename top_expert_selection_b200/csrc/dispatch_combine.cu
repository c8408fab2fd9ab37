// moe_dispatch / moe_combine: the row gathers around the grouped GEMM.
//
// Sources: Implementation:InternLM Lmdeploy Gemm MoeUtils -- Description
// (invokeMoeDispatch: tokens into expert-specific buffers; invokeMoeCombine:
// expert outputs back to token order, applying the routing scales), Usage
// Examples (gate -> dispatch -> grouped GEMM -> combine).
//
// Both are HBM-bound.  Work is token-major so each hidden row is read once:
// a warp owns a token row, moves it in 16-byte vectors with UNROLL vectors per
// lane in flight, and writes it to each of its k permuted rows (dispatch) or
// accumulates its k expert rows in fp32 in slot order (combine: acc = acc + w*x
// with a rounded product and a rounded add, then one RNE rounding to bf16).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kDcThreads = 256;
constexpr int kUnroll = 4;

struct DispatchArgs {
  const uint4* hidden;
  const int32_t* e2p;
  const int32_t* p2t;
  const int32_t* totals;
  uint4* out;
  int T, k;
  int vec_per_row;  // 16-byte vectors per row
  long long max_padded;
};

template <int KMAX>
__global__ void __launch_bounds__(kDcThreads) dispatch_kernel(DispatchArgs a) {
  pdl_entry();
  const int lane = threadIdx.x & 31;
  const long long warp_g = ((long long)blockIdx.x * kDcThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kDcThreads) >> 5;
  const long long P = min((long long)__ldg(&a.totals[0]), a.max_padded);
  const int V = a.vec_per_row;

  // token rows: read once, write k times
  for (long long t = warp_g; t < a.T; t += nwarps) {
    int dst[KMAX];
    const int k = a.k;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        const long long p = __ldg(&a.e2p[t * k + j]);
        dst[j] = (p >= 0 && p < P) ? (int)p : -1;
      }
    }
    // a token with no row here (every selection another shard's) is not read
    bool any = false;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) any |= (j < k && dst[j] >= 0);
    if (!any) continue;
    const uint4* src = a.hidden + t * V;
    for (int v0 = 0; v0 < V; v0 += 32 * kUnroll) {
      uint4 buf[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < V) buf[u] = __ldcs(src + v);
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k && dst[j] >= 0) {
          uint4* o = a.out + (long long)dst[j] * V;
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < V) o[v] = buf[u];
          }
        }
      }
    }
  }

  // padding rows below P: zero-filled
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (long long base = warp_g * 32; base < P; base += nwarps * 32) {
    const long long p = base + lane;
    const bool pad = p < P && __ldg(&a.p2t[p]) < 0;
    unsigned m = __ballot_sync(0xffffffffu, pad);
    while (m) {
      const int r = __ffs(m) - 1;
      m &= m - 1;
      uint4* o = a.out + (base + r) * V;
      for (int v = lane; v < V; v += 32) o[v] = z;
    }
  }
}

struct CombineArgs {
  const uint4* eo;
  long long eo_rows;  // rows of expert_out: a slot at or past it is skipped and recorded
  WsHeader* hdr;      // optional status word (NULL: not recorded)
  const int32_t* e2p;
  const void* weights;
  int weights_dtype;
  uint4* out;
  int T, k;
  int vec_per_row;
};

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// ELEMS = elements per 16-byte vector: 8 for bf16, 4 for fp32; KMAX bounds k
template <int ELEMS, int KMAX>
__global__ void __launch_bounds__(kDcThreads) combine_kernel(CombineArgs a) {
  pdl_entry();
  const int lane = threadIdx.x & 31;
  const long long warp_g = ((long long)blockIdx.x * kDcThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kDcThreads) >> 5;
  const int V = a.vec_per_row;
  for (long long t = warp_g; t < a.T; t += nwarps) {
    const int k = a.k;
    int src[KMAX];
    float w[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        src[j] = __ldg(&a.e2p[t * k + j]);
        w[j] = load_as_f32(a.weights, a.weights_dtype, (size_t)(t * k + j));
        if (src[j] >= a.eo_rows) {  // out of range: skipped (another shard's slots are -1)
          if (a.hdr && lane == 0) record_bounds(a.hdr);
          src[j] = -1;
        }
      }
    }
    for (int v0 = 0; v0 < V; v0 += 32 * kUnroll) {
      float acc[kUnroll][ELEMS];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
#pragma unroll
        for (int i = 0; i < ELEMS; ++i) acc[u][i] = 0.0f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k && src[j] >= 0) {
          const uint4* row = a.eo + (long long)src[j] * V;
          uint4 buf[kUnroll];
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < V) buf[u] = __ldcs(row + v);
          }
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            float x[ELEMS];
            if constexpr (ELEMS == 8) {
              unpack_bf16x8(buf[u], x);
            } else {
              x[0] = __uint_as_float(buf[u].x);
              x[1] = __uint_as_float(buf[u].y);
              x[2] = __uint_as_float(buf[u].z);
              x[3] = __uint_as_float(buf[u].w);
            }
            // fp32 accumulation in slot order: a rounded product, then a rounded add
#pragma unroll
            for (int i = 0; i < ELEMS; ++i) acc[u][i] = __fadd_rn(acc[u][i], __fmul_rn(w[j], x[i]));
          }
        }
      }
      uint4* o = a.out + t * V;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < V) {
          if constexpr (ELEMS == 8) {
            o[v] = pack_bf16x8(acc[u]);
          } else {
            o[v] = make_uint4(__float_as_uint(acc[u][0]), __float_as_uint(acc[u][1]), __float_as_uint(acc[u][2]),
                              __float_as_uint(acc[u][3]));
          }
        }
      }
    }
  }
}

int dc_grid(long long rows) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long warps = std::max(1LL, rows);
  const long long blocks = (warps * 32 + kDcThreads - 1) / kDcThreads;
  return (int)std::max(1LL, std::min<long long>(blocks, (long long)sms * (2048 / kDcThreads)));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_dispatch(int32_t T, int32_t H, int32_t k, int32_t dtype, const void* hidden,
                            const int32_t* expanded_to_permuted, const int32_t* permuted_to_token,
                            const int32_t* totals, int64_t max_padded, void* out, void* stream) {
  if (T < 0 || H <= 0 || k <= 0 || k > MOE_MAX_TOPK || max_padded < 0) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  const long long row_bytes = (long long)H * (dtype == MOE_BF16 ? 2 : 4);
  if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (!totals || (max_padded > 0 && (!out || !permuted_to_token)) || (T > 0 && (!hidden || !expanded_to_permuted)))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hidden) | reinterpret_cast<uintptr_t>(out)) & 15) return MOE_ERR_INVALID_ARG;
  if (max_padded > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  DispatchArgs a;
  a.hidden = reinterpret_cast<const uint4*>(hidden);
  a.e2p = expanded_to_permuted;
  a.p2t = permuted_to_token;
  a.totals = totals;
  a.out = reinterpret_cast<uint4*>(out);
  a.T = T;
  a.k = k;
  a.vec_per_row = (int)(row_bytes / 16);
  a.max_padded = max_padded;
  const int grid = dc_grid(std::max<long long>(T, (max_padded + 31) / 32));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (k <= 2)
    err = launch_pdl(dispatch_kernel<2>, dim3(grid), dim3(kDcThreads), 0, st, a);
  else if (k <= 8)
    err = launch_pdl(dispatch_kernel<8>, dim3(grid), dim3(kDcThreads), 0, st, a);
  else
    err = launch_pdl(dispatch_kernel<32>, dim3(grid), dim3(kDcThreads), 0, st, a);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_combine(int32_t T, int32_t H, int32_t k, int32_t dtype, const void* expert_out,
                           int64_t max_padded, const int32_t* expanded_to_permuted, const void* weights,
                           int32_t weights_dtype, void* out, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || H <= 0 || k <= 0 || k > MOE_MAX_TOPK || max_padded < 0) return MOE_ERR_INVALID_ARG;
  if (ws && ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (weights_dtype != MOE_BF16 && weights_dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  const long long row_bytes = (long long)H * (dtype == MOE_BF16 ? 2 : 4);
  if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if ((max_padded > 0 && !expert_out) || !expanded_to_permuted || !weights || !out) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(expert_out) | reinterpret_cast<uintptr_t>(out)) & 15) return MOE_ERR_INVALID_ARG;
  CombineArgs a;
  a.eo = reinterpret_cast<const uint4*>(expert_out);
  a.eo_rows = max_padded;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  a.e2p = expanded_to_permuted;
  a.weights = weights;
  a.weights_dtype = weights_dtype;
  a.out = reinterpret_cast<uint4*>(out);
  a.T = T;
  a.k = k;
  a.vec_per_row = (int)(row_bytes / 16);
  const int grid = dc_grid(T);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err;
  if (dtype == MOE_BF16) {
    if (k <= 2) err = launch_pdl(combine_kernel<8, 2>, dim3(grid), dim3(kDcThreads), 0, st, a);
    else if (k <= 8) err = launch_pdl(combine_kernel<8, 8>, dim3(grid), dim3(kDcThreads), 0, st, a);
    else err = launch_pdl(combine_kernel<8, 32>, dim3(grid), dim3(kDcThreads), 0, st, a);
  } else {
    if (k <= 2) err = launch_pdl(combine_kernel<4, 2>, dim3(grid), dim3(kDcThreads), 0, st, a);
    else if (k <= 8) err = launch_pdl(combine_kernel<4, 8>, dim3(grid), dim3(kDcThreads), 0, st, a);
    else err = launch_pdl(combine_kernel<4, 32>, dim3(grid), dim3(kDcThreads), 0, st, a);
  }
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
