// moe_ep_regroup: the receiving side of an expert-parallel (all-to-all-v)
// dispatch and the sending side of its return.
//
// Sources (by page title and section):
//   RMSNorm Router Top-K A2AV Kernel API Reference -- Background (the router's
//     top-k feeds the all-to-all-v MoE dispatch path);
//   flashinfer.fused_moe.trtllm_gen_routing -- Parameters (local_expert_offset,
//     local_num_experts: a rank owns a contiguous range of experts), Returns
//     (the tile-padded, expert-contiguous permuted layout);
//   Implementation:InternLM Lmdeploy Gemm MoeUtils -- invokeMoeDispatch /
//     invokeMoeCombine (rows gathered into expert buffers and back).
//
// World of W ranks, each owning L local experts.  counts[s][e] is the number
// of rows rank s sends for local expert e; the rows arrive in the receive
// buffer ordered by source rank, then expert, then the source's token order
// (what each rank's tile-1 route + dispatch produces for its destination's
// experts).  Regroup moves them into the tile-padded expert-contiguous layout
// ordered by expert, then source rank, then token -- the layout a single
// route of all ranks' tokens (concatenated in rank order) gives this rank's
// experts -- zeroes the padding rows and records for every padded row its
// receive row (-1 on padding).  Ungroup moves rows back from that layout to
// receive order (for the return all-to-all-v).
//
// Every block derives the plan (per-expert totals, padded offsets, and each
// (source, expert) run's receive and padded starts) from the counts in shared
// memory, then moves rows a warp each in 16-byte vectors (four loads in flight
// per lane before their stores).
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kEpThreads = 256;
constexpr int kEpMaxRuns = 8192;  // world * local experts
constexpr int kVec = 4;           // row copy: 16-byte vectors in flight per lane

struct EpArgs {
  const int32_t* counts;  // [W][L]
  int W, L, tile;
  int direction;          // 0: receive order -> padded, 1: padded -> receive order
  const uint4* src;
  uint4* dst;
  long long n_recv, max_padded;
  int vec_per_row;
  int32_t* offsets;       // [L + 1] (direction 0)
  int32_t* totals;        // [2] (direction 0)
  int32_t* p2r;           // [max_padded] (direction 0)
  WsHeader* hdr;          // optional status word
};

// shared plan: run r = s * L + e
struct EpPlan {
  int* recv_start;  // [W*L]
  int* pad_start;   // [W*L]
  int* cnt;         // [W*L]
  int* off;         // [L + 1]
  int* tot;         // [L]
};

__device__ void ep_plan(const EpArgs& a, EpPlan& p) {
  const int R = a.W * a.L;
  for (int r = threadIdx.x; r < R; r += blockDim.x) p.cnt[r] = max(0, a.counts[r]);
  __syncthreads();
  // per-expert totals and, per (s, e), the padded start within the expert
  for (int e = threadIdx.x; e < a.L; e += blockDim.x) {
    int run = 0;
    for (int s = 0; s < a.W; ++s) {
      p.pad_start[s * a.L + e] = run;  // relative to the expert's offset (added below)
      run += p.cnt[s * a.L + e];
    }
    p.tot[e] = run;
  }
  // per source s, the receive start of each of its runs (source-major order)
  if (threadIdx.x < 32) {
    // warp 0: exclusive scan of the counts in run order (lane l takes a chunk)
    const int lane = threadIdx.x;
    const int per = (R + 31) / 32, r0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (r0 + i < R) local += p.cnt[r0 + i];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i)
      if (r0 + i < R) {
        p.recv_start[r0 + i] = run;
        run += p.cnt[r0 + i];
      }
  }
  __syncthreads();
  // padded offsets over the experts (tile a power of two)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, tm = a.tile - 1;
    const int per = (a.L + 31) / 32, e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
      if (e0 + i < a.L) local += (p.tot[e0 + i] + tm) & ~tm;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int i = 0; i < per; ++i)
      if (e0 + i < a.L) {
        p.off[e0 + i] = run;
        run += (p.tot[e0 + i] + tm) & ~tm;
      }
    if (lane == 31) p.off[a.L] = incl;
  }
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x) p.pad_start[r] += p.off[r % a.L];
  __syncthreads();
}

__global__ void __launch_bounds__(kEpThreads) ep_regroup_kernel(EpArgs a) {
  extern __shared__ __align__(16) int eps[];
  const int R = a.W * a.L;
  EpPlan p;
  p.recv_start = eps;
  p.pad_start = eps + R;
  p.cnt = eps + 2 * R;
  p.off = eps + 3 * R;
  p.tot = eps + 3 * R + a.L + 1;
  pdl_entry();
  ep_plan(a, p);
  const int P = p.off[a.L];
  const long long n_recv = (long long)p.recv_start[R - 1] + p.cnt[R - 1];
  if (n_recv != a.n_recv || P > a.max_padded) {  // counts disagree with the buffers: nothing moves
    if (threadIdx.x == 0 && blockIdx.x == 0 && a.hdr) record_bounds(a.hdr);
    return;
  }
  if (a.direction == 0 && blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= a.L; e += blockDim.x) a.offsets[e] = p.off[e];
    if (threadIdx.x == 0) {
      a.totals[0] = P;
      a.totals[1] = P / a.tile;
    }
  }
  const int lane = threadIdx.x & 31;
  const long long warp_g = ((long long)blockIdx.x * kEpThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kEpThreads) >> 5;
  const int V = a.vec_per_row;
  // receive rows: the run holding row r (largest run with recv_start <= r and
  // a row), its padded row, one row per warp
  for (long long r = warp_g; r < a.n_recv; r += nwarps) {
    int lo = 0, hi = R - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.recv_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    // (a run with no rows shares its start with the next run, so the largest
    // run with start <= r < n_recv always has rows)
    const long long pr = (long long)p.pad_start[lo] + (r - p.recv_start[lo]);
    const uint4* __restrict__ s = a.direction == 0 ? a.src + r * V : a.src + pr * V;
    uint4* __restrict__ d = a.direction == 0 ? a.dst + pr * V : a.dst + r * V;
    // kVec 16-byte loads in flight per lane before their stores
    for (int v0 = lane; v0 < V; v0 += 32 * kVec) {
      uint4 t[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u)
        if (v0 + 32 * u < V) t[u] = __ldcs(s + v0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kVec; ++u)
        if (v0 + 32 * u < V) __stcs(d + v0 + 32 * u, t[u]);
    }
    if (a.direction == 0 && lane == 0) a.p2r[pr] = (int32_t)r;
  }
  // padding rows (direction 0): zero, receive row -1; a warp per padded row,
  // spread over the whole grid (the padded row's expert is the largest with
  // off[e] <= row, so experts without rows are passed over)
  if (a.direction == 0) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (long long row = warp_g; row < P; row += nwarps) {
      int lo = 0, hi = a.L - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.off[mid] <= row) lo = mid; else hi = mid - 1;
      }
      if (row < (long long)p.off[lo] + p.tot[lo]) continue;  // a received row, moved above
      for (int v = lane; v < V; v += 32) __stcs(a.dst + row * V + v, z);
      if (lane == 0) a.p2r[row] = -1;
    }
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_ep_regroup(int32_t world, int32_t local_experts, int32_t H, int32_t dtype, int32_t tile,
                              const int32_t* counts, int32_t direction, void* recv, int64_t n_recv,
                              void* padded, int64_t max_padded, int32_t* padded_offsets, int32_t* totals,
                              int32_t* padded_to_recv, void* ws, size_t ws_bytes, void* stream) {
  if (world <= 0 || local_experts <= 0 || H <= 0 || n_recv < 0 || max_padded < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)world * local_experts > kEpMaxRuns) return MOE_ERR_UNSUPPORTED;
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (tile <= 0 || (tile & (tile - 1)) != 0 || tile > 4096) return MOE_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return MOE_ERR_INVALID_ARG;
  const long long row_bytes = (long long)H * (dtype == MOE_BF16 ? 2 : 4);
  if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (!counts || (n_recv > 0 && !recv) || (max_padded > 0 && !padded)) return MOE_ERR_INVALID_ARG;
  if (direction == 0 && (!padded_offsets || !totals || (max_padded > 0 && !padded_to_recv))) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(recv) | reinterpret_cast<uintptr_t>(padded)) & 15) return MOE_ERR_INVALID_ARG;
  if (ws && ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  if (n_recv > 0x7fffffffLL || max_padded > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  EpArgs a;
  a.counts = counts;
  a.W = world;
  a.L = local_experts;
  a.tile = tile;
  a.direction = direction;
  a.src = reinterpret_cast<const uint4*>(direction == 0 ? recv : padded);
  a.dst = reinterpret_cast<uint4*>(direction == 0 ? padded : recv);
  a.n_recv = n_recv;
  a.max_padded = max_padded;
  a.vec_per_row = (int)(row_bytes / 16);
  a.offsets = padded_offsets;
  a.totals = totals;
  a.p2r = padded_to_recv;
  a.hdr = reinterpret_cast<WsHeader*>(ws);
  const int R = world * local_experts;
  const size_t smem = (size_t)(3 * R + 2 * local_experts + 1) * 4;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long warps = std::max<long long>(n_recv, max_padded);
  const int grid = (int)std::max(1LL, std::min<long long>((warps * 32 + kEpThreads - 1) / kEpThreads, 4LL * sms));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(ep_regroup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const cudaError_t e = launch_pdl(ep_regroup_kernel, dim3(grid), dim3(kEpThreads), smem, st, a);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
