// Combine (h'_t = u_t + FFN^(s)(u_t) + sum_k g_{t,k} FFN^(r)(u_t)), the
// auxiliary-loss-free bias update ("DeepSeek-V3 Teknik Raporu", Yöntem 2), and
// the library's error-word entry points.
#include "host.cuh"

namespace moe {

// One block per token; each thread handles 8 consecutive channels (16 bytes
// of bf16 from u, the shared row and every routed row) per step, all the
// step's loads issued before the sums. FP32 sum in the fixed order: u,
// shared, k = 0..K-1.
constexpr int COMBINE_KMAX = 16;

__device__ __forceinline__ void bf16x8_to_float(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFF);
    f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}

// Eight values of a row as floats: bf16 (one 16-byte load) or FP32 (two).
template <typename Y>
struct Row8;
template <>
struct Row8<uint16_t> {
  uint4 v;
  __device__ __forceinline__ void load(const uint16_t* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void get(float (&f)[8]) const { bf16x8_to_float(v, f); }
};
template <>
struct Row8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p + 4));
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

template <typename Y>
__global__ void __launch_bounds__(128) combine_kernel(const uint16_t* __restrict__ u,
                                                      const Y* __restrict__ y_perm,
                                                      const Y* __restrict__ y_shared,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gates, int K,
                                                      int d, int P, uint16_t* out) {
  __shared__ int s_row[COMBINE_KMAX];
  __shared__ float s_g[COMBINE_KMAX];
  const int t = blockIdx.x;
  if (threadIdx.x < K) {
    int r = inv[static_cast<size_t>(t) * K + threadIdx.x];
    if (r < 0 || r >= P) {
      set_device_error(MOE_ERR_INVALID_ARG);
      r = -1;
    }
    s_row[threadIdx.x] = r;
    s_g[threadIdx.x] = gates[static_cast<size_t>(t) * K + threadIdx.x];
  }
  __syncthreads();
  const size_t base = static_cast<size_t>(t) * d;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    const uint4 a = *reinterpret_cast<const uint4*>(u + base + c);
    Row8<Y> sh;
    sh.load(y_shared + base + c);
    Row8<Y> yv[COMBINE_KMAX];
#pragma unroll
    for (int k = 0; k < COMBINE_KMAX; ++k) {
      yv[k].zero();
      if (k < K && s_row[k] >= 0) yv[k].load(y_perm + static_cast<size_t>(s_row[k]) * d + c);
    }
    float acc[8], f[8];
    bf16x8_to_float(a, acc);
    sh.get(f);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += f[i];
#pragma unroll
    for (int k = 0; k < COMBINE_KMAX; ++k) {
      if (k >= K || s_row[k] < 0) continue;
      const float g = s_g[k];
      yv[k].get(f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[i], acc[i]);
    }
    uint4 o;
    o.x = float_to_bf16_bits(acc[0]) | (static_cast<uint32_t>(float_to_bf16_bits(acc[1])) << 16);
    o.y = float_to_bf16_bits(acc[2]) | (static_cast<uint32_t>(float_to_bf16_bits(acc[3])) << 16);
    o.z = float_to_bf16_bits(acc[4]) | (static_cast<uint32_t>(float_to_bf16_bits(acc[5])) << 16);
    o.w = float_to_bf16_bits(acc[6]) | (static_cast<uint32_t>(float_to_bf16_bits(acc[7])) << 16);
    *reinterpret_cast<uint4*>(out + base + c) = o;
  }
}

// One block: b_i -= gamma if counts_i * N_r > T*K_r, b_i += gamma if below,
// unchanged if equal (FP32 arithmetic). Also max_i counts_i * N_r / (T*K_r).
__global__ void __launch_bounds__(1024) bias_update_kernel(float* b, const int32_t* __restrict__ counts,
                                                           int N_r, long long mean_load_x_nr,
                                                           float gamma, float* max_over_mean) {
  __shared__ int s_max[32];
  int local_max = 0;
  for (int i = threadIdx.x; i < N_r; i += blockDim.x) {
    const int c = counts[i];
    const long long load = static_cast<long long>(c) * N_r;
    if (load > mean_load_x_nr)
      b[i] = b[i] - gamma;
    else if (load < mean_load_x_nr)
      b[i] = b[i] + gamma;
    local_max = max(local_max, c);
  }
  if (max_over_mean == nullptr) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local_max = max(local_max, __shfl_xor_sync(0xffffffffu, local_max, o));
  if (lane_id() == 0) s_max[threadIdx.x >> 5] = local_max;
  __syncthreads();
  if (threadIdx.x == 0) {
    int m = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = max(m, s_max[w]);
    *max_over_mean = mean_load_x_nr > 0
                         ? static_cast<float>(static_cast<double>(m) * N_r / static_cast<double>(mean_load_x_nr))
                         : 0.0f;
  }
}

// Waits on an mbarrier nothing signals; gives up after limit_ns.
__global__ void wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace moe

template <typename Y>
static int combine(const uint16_t* u, const Y* y_perm, const Y* y_shared, const int32_t* inv, const float* gates,
                   int T, int K_r, int d, uint16_t* out, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(T >= 0 && K_r >= 1 && d >= 0);
  MOE_CHECK_SUPPORTED(K_r <= 16 && d % 8 == 0);
  if (T == 0 || d == 0) return MOE_OK;
  MOE_CHECK_ARG(u && y_perm && y_shared && inv && gates && out);
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(u) % 16 == 0 && reinterpret_cast<uintptr_t>(y_perm) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(y_shared) % 16 == 0 && reinterpret_cast<uintptr_t>(out) % 16 == 0);
  MOE_CHECK_SUPPORTED(static_cast<long long>(T) * K_r < (1LL << 31));
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  combine_kernel<Y><<<T, 128, 0, as_stream(stream)>>>(u, y_perm, y_shared, inv, gates, K_r, d, T * K_r, out);
  return launch_status();
}

extern "C" int moe_combine(const uint16_t* u, const uint16_t* y_perm, const uint16_t* y_shared,
                           const int32_t* inv, const float* gates, int T, int K_r, int d,
                           uint16_t* out, void* stream) {
  return combine(u, y_perm, y_shared, inv, gates, T, K_r, d, out, stream);
}

extern "C" int moe_combine_fp32(const uint16_t* u, const float* y_perm, const float* y_shared,
                                const int32_t* inv, const float* gates, int T, int K_r, int d,
                                uint16_t* out, void* stream) {
  return combine(u, y_perm, y_shared, inv, gates, T, K_r, d, out, stream);
}

extern "C" int moe_bias_update(float* b, const int32_t* counts, int N_r, int T, int K_r, float gamma,
                               float* max_over_mean_out, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(N_r >= 1 && T >= 0 && K_r >= 1 && b && counts);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  bias_update_kernel<<<1, 1024, 0, as_stream(stream)>>>(b, counts, N_r, static_cast<long long>(T) * K_r,
                                                        gamma, max_over_mean_out);
  return launch_status();
}

extern "C" int moe_debug_wait_timeout(int timeout_us, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(timeout_us >= 1 && timeout_us <= 1000000);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  wait_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  return launch_status();
}

extern "C" int moe_get_error(int* device_status) {
  using namespace moe;
  MOE_CHECK_ARG(device_status);
  if (int st = cuda_status(cudaDeviceSynchronize(), "moe_get_error: synchronize")) return st;
  int v = 0;
  if (int st = cuda_status(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)), "moe_get_error: read"))
    return st;
  const int zero = 0;
  if (int st = cuda_status(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)), "moe_get_error: clear"))
    return st;
  *device_status = v;
  return MOE_OK;
}

extern "C" const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE";
    default: return "unknown moe_status";
  }
}

extern "C" int moe_version(void) { return 200; }

extern "C" const char* moe_last_error_detail(void) { return moe::last_error_buf(); }
