// Stable counting sort of (token, expert) pairs by expert: histogram, prefix
// sum, scatter. Row order of the result is (expert ascending, token
// ascending), identical to a stable sort; the FP8 rows and their 1x128 scales
// are then gathered into that order for the grouped GEMM.
//
// Four launches:
//   count   - one block per 256 tokens: per-warp bitmasks of which lanes
//             (tokens) chose each expert; the block's count per expert.
//   scan    - one block: counts, offsets, and each block's base row per expert.
//   scatter - same blocks as count: row = base + rank of the token among the
//             block's earlier tokens with the same expert.
//   gather  - one warp per row: copies the FP8 row and its scales.
#include "host.cuh"

namespace moe {
namespace perm {

constexpr int TOK = 256;        // tokens per block (one per thread)
constexpr int WARPS = TOK / 32;

// Bitmask per (warp, expert) of the lanes whose token selected the expert.
__device__ __forceinline__ void build_masks(uint32_t* masks, const int32_t* __restrict__ topk,
                                            int T, int K, int N_r, int t) {
  const int w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < WARPS * N_r; i += TOK) masks[i] = 0u;
  __syncthreads();
  if (t < T) {
    const uint32_t bit = 1u << lane_id();
    for (int k = 0; k < K; ++k) {
      const int e = topk[static_cast<size_t>(t) * K + k];
      if (e < 0 || e >= N_r) {
        set_device_error(MOE_ERR_INVALID_ARG);
        continue;
      }
      atomicOr(&masks[w * N_r + e], bit);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(TOK) count_kernel(const int32_t* __restrict__ topk, int T, int K,
                                                    int N_r, int32_t* __restrict__ block_count) {
  extern __shared__ uint32_t masks[];
  const int t = blockIdx.x * TOK + threadIdx.x;
  build_masks(masks, topk, T, K, N_r, t);
  for (int e = threadIdx.x; e < N_r; e += TOK) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) c += __popc(masks[w * N_r + e]);
    block_count[static_cast<size_t>(blockIdx.x) * N_r + e] = c;
  }
}

// One block of 1024 threads; thread e owns expert e (N_r <= 1024).
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ block_count,
                                                    int n_blocks, int N_r,
                                                    int32_t* __restrict__ block_base,
                                                    int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_sum[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < N_r)
    for (int b = 0; b < n_blocks; ++b) total += block_count[static_cast<size_t>(b) * N_r + e];
  // exclusive scan of `total` over experts
  int incl = total;
  const int lane = lane_id();
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[threadIdx.x >> 5] = incl;
  __syncthreads();
  if (threadIdx.x < 32) {
    int ws = warp_sum[lane];
    int wincl = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += v;
    }
    warp_sum[lane] = wincl - ws;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - total + warp_sum[threadIdx.x >> 5];
  if (e < N_r) {
    counts[e] = total;
    offsets[e] = excl;
    if (e == N_r - 1) offsets[N_r] = excl + total;
    int run = excl;
    for (int b = 0; b < n_blocks; ++b) {
      block_base[static_cast<size_t>(b) * N_r + e] = run;
      run += block_count[static_cast<size_t>(b) * N_r + e];
    }
  }
}

__global__ void __launch_bounds__(TOK) scatter_kernel(const int32_t* __restrict__ topk, int T,
                                                      int K, int N_r,
                                                      const int32_t* __restrict__ block_base,
                                                      int32_t* __restrict__ sorted_token,
                                                      int32_t* __restrict__ inv) {
  extern __shared__ uint32_t masks[];
  const int t = blockIdx.x * TOK + threadIdx.x;
  build_masks(masks, topk, T, K, N_r, t);
  if (t >= T) return;
  const int w = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane_id()) - 1u;
  for (int k = 0; k < K; ++k) {
    const int e = topk[static_cast<size_t>(t) * K + k];
    if (e < 0 || e >= N_r) {   // the error is recorded by count_kernel
      inv[static_cast<size_t>(t) * K + k] = -1;
      continue;
    }
    int rank = __popc(masks[w * N_r + e] & lt);
    for (int w2 = 0; w2 < w; ++w2) rank += __popc(masks[w2 * N_r + e]);
    const int row = block_base[static_cast<size_t>(blockIdx.x) * N_r + e] + rank;
    sorted_token[row] = t;
    inv[static_cast<size_t>(t) * K + k] = row;
  }
}

// One warp per destination row: d bytes of codes as 16-byte vectors, then the
// d/128 scales.
// Row moves in token order: a warp reads token t's code row (and its
// scales) once and writes it to the K_r permuted rows inv[t][0..K_r). In
// permuted order the same token row would be read K_r times, by warps far
// apart in time, and mostly from DRAM again (L2 does not hold the whole of
// xq between its uses). The row goes through registers in chunks of up to
// GV x 16 bytes per lane, all loads of a chunk issued before its stores.
constexpr int GV = 8;

__global__ void __launch_bounds__(256) gather_kernel(const int32_t* __restrict__ inv, int T, int K,
                                                     long long P, const uint8_t* __restrict__ xq,
                                                     const float* __restrict__ xs, int d,
                                                     uint8_t* __restrict__ xq_perm,
                                                     float* __restrict__ xs_perm) {
  const int lane = lane_id();
  const int nvec = d / 16;
  const int ns = d / 128;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += warps) {
    const uint4* src = reinterpret_cast<const uint4*>(xq + static_cast<size_t>(t) * d);
    for (int base = 0; base < nvec; base += 32 * GV) {
      uint4 v[GV];
#pragma unroll
      for (int j = 0; j < GV; ++j) {
        const int i = base + j * 32 + lane;
        if (i < nvec) v[j] = __ldg(src + i);
      }
      for (int k = 0; k < K; ++k) {
        const long long p = inv[t * K + k];
        if (p < 0 || p >= P) continue;   // only after an invalid expert index (error already set)
        uint4* dst = reinterpret_cast<uint4*>(xq_perm + static_cast<size_t>(p) * d);
#pragma unroll
        for (int j = 0; j < GV; ++j) {
          const int i = base + j * 32 + lane;
          if (i < nvec) dst[i] = v[j];
        }
      }
    }
    for (int i = lane; i < ns; i += 32) {
      const float sc = __ldg(xs + static_cast<size_t>(t) * ns + i);
      for (int k = 0; k < K; ++k) {
        const long long p = inv[t * K + k];
        if (p >= 0 && p < P) xs_perm[static_cast<size_t>(p) * ns + i] = sc;
      }
    }
  }
}

}  // namespace perm
}  // namespace moe

extern "C" size_t moe_permute_workspace(int T, int N_r) {
  if (T <= 0 || N_r <= 0) return 0;
  const size_t nb = (static_cast<size_t>(T) + moe::perm::TOK - 1) / moe::perm::TOK;
  return 2 * nb * static_cast<size_t>(N_r) * sizeof(int32_t);
}

extern "C" int moe_permute(const int32_t* topk_idx, int T, int K_r, int N_r, const uint8_t* xq,
                           const float* xs, int d, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_token, int32_t* inv, uint8_t* xq_perm, float* xs_perm,
                           void* workspace, size_t ws_bytes, void* stream) {
  using namespace moe;
  using namespace moe::perm;
  MOE_CHECK_ARG(T >= 0 && K_r >= 1 && N_r >= 1);
  MOE_CHECK_SUPPORTED(N_r <= 1024 && K_r <= 16 && K_r <= N_r);
  MOE_CHECK_ARG(counts && offsets);
  const bool move_rows = xq != nullptr;
  if (move_rows) {
    MOE_CHECK_ARG(xs && xq_perm && xs_perm && d > 0);
    MOE_CHECK_SUPPORTED(d % 128 == 0);
    MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(xq) % 16 == 0 && reinterpret_cast<uintptr_t>(xq_perm) % 16 == 0);
  }
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  cudaStream_t s = as_stream(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, N_r * sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(offsets, 0, (N_r + 1) * sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  MOE_CHECK_ARG(topk_idx && sorted_token && inv && workspace);
  MOE_CHECK_ARG(ws_bytes >= moe_permute_workspace(T, N_r));
  const int nb = (T + TOK - 1) / TOK;
  int32_t* block_count = static_cast<int32_t*>(workspace);
  int32_t* block_base = block_count + static_cast<size_t>(nb) * N_r;
  const size_t sh = static_cast<size_t>(WARPS) * N_r * sizeof(uint32_t);
  count_kernel<<<nb, TOK, sh, s>>>(topk_idx, T, K_r, N_r, block_count);
  scan_kernel<<<1, 1024, 0, s>>>(block_count, nb, N_r, block_base, counts, offsets);
  scatter_kernel<<<nb, TOK, sh, s>>>(topk_idx, T, K_r, N_r, block_base, sorted_token, inv);
  if (move_rows) {
    const long long P = static_cast<long long>(T) * K_r;
    long long blocks = (static_cast<long long>(T) + 7) / 8;       // a warp per token
    const long long cap = static_cast<long long>(di.sm_count) * 8;  // one resident wave
    if (blocks > cap) blocks = cap;
    gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(inv, T, K_r, P, xq, xs, d, xq_perm, xs_perm);
  }
  return launch_status();
}
