// Router: s_{i,t} = Sigmoid(u_t . e_i), biased top-K_r selection, normalised
// gates ("DeepSeek-V3 Teknik Raporu", Yöntem 2; "DeepSeek-V3 Technical
// Report" (fr), Méthode 2).
//
// The logits are a [T x d] x [d x N_r] product: one CTA takes 128 tokens and
// all N_r experts, streams u and e through shared memory with TMA (128-byte
// swizzled K blocks of 64 bf16), and accumulates u . e^T in TMEM with
// tcgen05 kind::f16 MMAs (BF16 inputs, FP32 accumulation). Four epilogue
// warps then own one token row each (one TMEM lane) and do sigmoid, the
// biased top-K and the gates in registers.
#include "host.cuh"

namespace moe {
namespace route {

constexpr int BM = 128;          // tokens per CTA (TMEM lanes)
constexpr int BK = 64;           // bf16 per K block = 128 bytes = one swizzle row
constexpr int STAGES = 4;
constexpr int THREADS = 192;     // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int A_BYTES = BM * BK * 2;

// Inserts (key, idx, s) into a list sorted by key descending; candidates
// arrive in increasing idx, so a candidate never passes an equal key (equal
// keys keep the lower index first). Once a slot is taken, the rest of the
// list shifts down by one.
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&kk)[KMAX], int (&ii)[KMAX], float (&ss)[KMAX],
                                            float key, int idx, float s) {
  bool shifting = false;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const bool take = shifting || (key > kk[j]);
    if (take) {
      const float tk = kk[j];
      const int ti = ii[j];
      const float ts = ss[j];
      kk[j] = key;
      ii[j] = idx;
      ss[j] = s;
      key = tk;
      idx = ti;
      s = ts;
      shifting = true;
    }
  }
}

template <int KMAX>
__device__ __forceinline__ void topk_init(float (&kk)[KMAX], int (&ii)[KMAX], float (&ss)[KMAX]) {
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    kk[j] = -INFINITY;
    ii[j] = 0x7fffffff;
    ss[j] = 0.0f;
  }
}

// Gates g_k = s_k / sum_{k'<K} s_k' (sum in k order, FP32, IEEE division).
template <int KMAX>
__device__ __forceinline__ void topk_store(const int (&ii)[KMAX], const float (&ss)[KMAX], int K,
                                           int32_t* idx_out, float* gate_out) {
  float sum = 0.0f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < K) sum += ss[j];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < K) {
      idx_out[j] = ii[j];
      gate_out[j] = __fdiv_rn(ss[j], sum);
    }
  }
}

__device__ __forceinline__ float sigmoidf(float z) { return __fdiv_rn(1.0f, 1.0f + expf(-z)); }

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float bias[256];
};

template <int KMAX>
__global__ void __launch_bounds__(THREADS, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_e,
                  const float* __restrict__ b, int T, int d, int N_r, int NP, int K,
                  float* __restrict__ scores_out, int32_t* __restrict__ topk_idx,
                  float* __restrict__ gates, uint32_t tmem_cols) {
  extern __shared__ uint8_t smem_raw[];
  // operand tiles need 1024-byte alignment for the 128-byte swizzle
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int b_bytes = NP * BK * 2;
  const int stage_bytes = A_BYTES + b_bytes;
  Smem& sm = *reinterpret_cast<Smem*>(tiles + STAGES * stage_bytes);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int tile = blockIdx.x;
  const int KB = d / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_u);
    tma_prefetch_desc(&tm_e);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, tmem_cols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < N_r; i += THREADS) sm.bias[i] = b[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      // producer: K blocks of u (128 x 64) and e (NP x 64)
      int armed_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) armed_parity[s] = -1;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&sm.empty[s], ph ^ 1, abort)) break;
        uint8_t* a_dst = tiles + s * stage_bytes;
        mbar_arrive_expect_tx(&sm.full[s], stage_bytes);
        tma_load_2d(a_dst, &tm_u, &sm.full[s], kb * BK, tile * BM);
        tma_load_2d(a_dst + A_BYTES, &tm_e, &sm.full[s], kb * BK, 0);
        armed_parity[s] = ph;
      }
      if (*abort) {
        // let every issued copy land before the block's shared memory is released
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (armed_parity[s] >= 0) mbar_wait(&sm.full[s], armed_parity[s], &never, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(1, 1, BM, NP);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&sm.full[s], ph, abort)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + s * stage_bytes);
        const uint64_t ad = sw128_kmajor_desc(a_addr);
        const uint64_t bd = sw128_kmajor_desc(a_addr + A_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)  // 16 bf16 = 32 bytes per MMA
          umma_f16(tmem, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0);
        umma_commit(&sm.empty[s]);
      }
      umma_commit(&sm.acc_full);
      // all MMAs of this thread complete before TMEM is released
      umma_commit(&sm.drain);
      volatile int never = 0;
      mbar_wait(&sm.drain, 0, &never, 100000000ull);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int t = tile * BM + r;
    if (warp_wait(&sm.acc_full, 0, abort)) {
      tc_fence_after();
      float kk[KMAX], ss[KMAX];
      int ii[KMAX];
      topk_init(kk, ii, ss);
      for (int c0 = 0; c0 < NP; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = c0 + j;
          if (col < N_r) {
            const float s = sigmoidf(v[j]);
            v[j] = s;
            topk_insert(kk, ii, ss, s + sm.bias[col], col, s);
          }
        }
        if (scores_out != nullptr && t < T) {
          float* dst = scores_out + static_cast<size_t>(t) * N_r + c0;
          const int ncol = min(32, N_r - c0);
          if ((N_r & 3) == 0 && ncol == 32) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
            for (int j = 0; j < ncol; ++j) dst[j] = v[j];
          }
        }
      }
      if (t < T) topk_store(ii, ss, K, topk_idx + static_cast<size_t>(t) * K, gates + static_cast<size_t>(t) * K);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Top-K from given FP32 affinities: one thread per token.
template <int KMAX>
__global__ void __launch_bounds__(128)
    route_from_scores_kernel(const float* __restrict__ scores, const float* __restrict__ b, int T,
                             int N_r, int K, float* __restrict__ scores_out,
                             int32_t* __restrict__ topk_idx, float* __restrict__ gates) {
  extern __shared__ float s_bias[];
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) s_bias[i] = b[i];
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float kk[KMAX], ss[KMAX];
  int ii[KMAX];
  topk_init(kk, ii, ss);
  const float* row = scores + static_cast<size_t>(t) * N_r;
  for (int i = 0; i < N_r; ++i) {
    const float s = row[i];
    if (scores_out) scores_out[static_cast<size_t>(t) * N_r + i] = s;
    topk_insert(kk, ii, ss, s + s_bias[i], i, s);
  }
  topk_store(ii, ss, K, topk_idx + static_cast<size_t>(t) * K, gates + static_cast<size_t>(t) * K);
}

}  // namespace route
}  // namespace moe

extern "C" int moe_route(const uint16_t* u, const uint16_t* e, const float* b,
                         const float* scores_in, int T, int d, int N_r, int K_r,
                         float* scores_out, int32_t* topk_idx, float* gates, void* stream) {
  using namespace moe;
  using namespace moe::route;
  MOE_CHECK_ARG(T >= 0 && d >= 0 && N_r >= 1 && K_r >= 1);
  MOE_CHECK_SUPPORTED(K_r <= 16 && K_r <= N_r && N_r <= 256);
  if (T == 0) return MOE_OK;
  MOE_CHECK_ARG(b && topk_idx && gates);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  cudaStream_t s = as_stream(stream);
  if (scores_in != nullptr) {
    const int blocks = (T + 127) / 128;
    const size_t sh = N_r * sizeof(float);
    if (K_r <= 8)
      route_from_scores_kernel<8><<<blocks, 128, sh, s>>>(scores_in, b, T, N_r, K_r, scores_out, topk_idx, gates);
    else
      route_from_scores_kernel<16><<<blocks, 128, sh, s>>>(scores_in, b, T, N_r, K_r, scores_out, topk_idx, gates);
    return launch_status();
  }
  MOE_CHECK_ARG(u && e && d > 0);
  MOE_CHECK_SUPPORTED(d % BK == 0);
  const int NP = ((N_r + 15) / 16) * 16;
  uint32_t tmem_cols = 32;
  while (static_cast<int>(tmem_cols) < NP) tmem_cols *= 2;
  CUtensorMap tm_u, tm_e;
  if (int st = make_tmap_2d(&tm_u, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, d, BM, BK)) return st;
  if (int st = make_tmap_2d(&tm_e, e, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N_r, d, NP, BK)) return st;
  const size_t smem = 1024 + STAGES * (A_BYTES + NP * BK * 2) + sizeof(Smem);
  const int blocks = (T + BM - 1) / BM;
  if (K_r <= 8) {
    auto k = router_kernel<8>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<blocks, THREADS, smem, s>>>(tm_u, tm_e, b, T, d, N_r, NP, K_r, scores_out, topk_idx, gates, tmem_cols);
  } else {
    auto k = router_kernel<16>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    k<<<blocks, THREADS, smem, s>>>(tm_u, tm_e, b, T, d, N_r, NP, K_r, scores_out, topk_idx, gates, tmem_cols);
  }
  return launch_status();
}
