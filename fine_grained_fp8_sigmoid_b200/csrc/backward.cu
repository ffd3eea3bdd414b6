// The expert FFN's backward in the FP8 scheme: the elementwise and layout
// steps around the backward's GEMMs (which run on the grouped GEMM kernel,
// moe_grouped_scaled_gemm_fp8).
//
// The pages train in FP8 ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8
// bullet: E4M3 on all tensors, activations in 1x128 tiles, weights in
// 128x128 blocks) and print no backward details. An operand's granularity
// follows its role in the product: the operand whose rows are the product's
// rows gets one FP32 scale per 1x128 tile along the contraction, the other one
// per 128x128 block. wgrad contracts over the expert's tokens, so its operands
// are the transposes of token-major tensors, quantised along the tokens:
//
//   moe_swiglu_backward_quant - dG = dH U silu'(G), dU = dH silu(G), then
//                               [dG | dU] in 1x128 tiles (dgrad's operand)
//   moe_quant_1x128_t         - a token-major FP32 or BF16 tensor, per group of
//                               rows, transposed and quantised in 1x128 tiles
//                               along the tokens (wgrad's activation role)
//   moe_quant_128x128_t       - FP8 rows with 1x128 scales (the forward's X or
//                               H), dequantised, transposed and requantised in
//                               128x128 blocks (wgrad's weight role)
//   moe_transpose             - 1- or 4-byte matrices transposed into a column
//                               range of the destination: the weights' codes
//                               and block scales for dgrad (a 128x128 block
//                               stays one block under transposition)
#include "host.cuh"

namespace moe {
namespace bwd {

// sigma(x) with the IEEE exponential and division
__device__ __forceinline__ float sigmoid_rn(float x) { return __fdiv_rn(1.0f, 1.0f + expf(-x)); }

// One warp per (row, 128-column tile of I): lane l owns columns 4l..4l+3 of
// the tile in dG and in dU; each of the two 1x128 tiles gets its scale.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(const float* __restrict__ g, const float* __restrict__ u,
                                                              const float* __restrict__ dh, int R, int I,
                                                              float* __restrict__ dgu, uint8_t* __restrict__ q,
                                                              float* __restrict__ qs) {
  const int lane = lane_id();
  const int tiles = I / 128;
  const long long n = static_cast<long long>(R) * tiles;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long w = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); w < n; w += warps) {
    const long long r = w / tiles;
    const int j = static_cast<int>(w - r * tiles);
    const size_t in = static_cast<size_t>(r) * I + j * 128 + lane * 4;
    const float4 gv = __ldg(reinterpret_cast<const float4*>(g + in));
    const float4 uv = __ldg(reinterpret_cast<const float4*>(u + in));
    const float4 hv = __ldg(reinterpret_cast<const float4*>(dh + in));
    const float G[4] = {gv.x, gv.y, gv.z, gv.w}, U[4] = {uv.x, uv.y, uv.z, uv.w}, D[4] = {hv.x, hv.y, hv.z, hv.w};
    float dg[4], du[4], mg = 0.0f, mu = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float s = sigmoid_rn(G[i]);
      const float silu = G[i] * s;
      dg[i] = D[i] * U[i] * (s * (1.0f + G[i] * (1.0f - s)));
      du[i] = D[i] * silu;
      mg = fmaxf(mg, fabsf(dg[i]));
      mu = fmaxf(mu, fabsf(du[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
      mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, o));
    }
    const float sg = tile_scale(mg), su = tile_scale(mu);
    const size_t og = static_cast<size_t>(r) * 2 * I + j * 128 + lane * 4;   // dG half of the row
    const size_t ou = og + I;                                                 // dU half
    if (dgu != nullptr) {
      *reinterpret_cast<float4*>(dgu + og) = make_float4(dg[0], dg[1], dg[2], dg[3]);
      *reinterpret_cast<float4*>(dgu + ou) = make_float4(du[0], du[1], du[2], du[3]);
    }
    const uint32_t cg = e4m3x2(__fdiv_rn(dg[0], sg), __fdiv_rn(dg[1], sg)) |
                        (e4m3x2(__fdiv_rn(dg[2], sg), __fdiv_rn(dg[3], sg)) << 16);
    const uint32_t cu = e4m3x2(__fdiv_rn(du[0], su), __fdiv_rn(du[1], su)) |
                        (e4m3x2(__fdiv_rn(du[2], su), __fdiv_rn(du[3], su)) << 16);
    *reinterpret_cast<uint32_t*>(q + og) = cg;
    *reinterpret_cast<uint32_t*>(q + ou) = cu;
    if (lane == 0) {
      qs[static_cast<size_t>(r) * (2 * tiles) + j] = sg;
      qs[static_cast<size_t>(r) * (2 * tiles) + tiles + j] = su;
    }
  }
}

// Group of a row block: dst_off[g] <= p * 128 < dst_off[g + 1].
__device__ __forceinline__ int block_group(const int32_t* dst_off, int n_groups, int row0) {
  int lo = 0, hi = n_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(dst_off + mid) <= row0) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One block of 128 threads per (128 tokens, 128 columns): the tile is staged
// in shared memory as [token][column]; thread c then owns column c: its 128
// token values form one 1x128 tile of the transposed tensor (KIND 0: FP32
// input, KIND 1: BF16 input; a scale per column and token block) or belong to
// one 128x128 block (KIND 2: FP8 input with 1x128 scales; one scale for the
// whole tile).
template <int KIND>
__global__ void __launch_bounds__(128) quant_t_kernel(const void* __restrict__ x, const float* __restrict__ xs,
                                                      int ld, int cols, const int32_t* __restrict__ src_off,
                                                      const int32_t* __restrict__ dst_off, int n_groups, int Ktot,
                                                      uint8_t* __restrict__ q, float* __restrict__ s) {
  extern __shared__ float tile[];                    // [128][129]
  __shared__ float red[4];
  const int p = blockIdx.x;                          // token block of the output's K
  const int cb = blockIdx.y;                         // column block
  const int g = block_group(dst_off, n_groups, p * 128);
  const int d0 = __ldg(dst_off + g), Kg = __ldg(dst_off + g + 1) - d0;   // the group's padded token count
  const int first = __ldg(src_off + g) + (p * 128 - d0);
  const int live = max(0, min(128, __ldg(src_off + g + 1) - first));
  const int c = threadIdx.x;
  for (int t = 0; t < 128; ++t) {
    float v = 0.0f;
    if (t < live) {
      const size_t at = static_cast<size_t>(first + t) * ld + cb * 128 + c;
      if (KIND == 0) {
        v = __ldg(static_cast<const float*>(x) + at);
      } else if (KIND == 1) {
        v = bf16_bits_to_float(__ldg(static_cast<const uint16_t*>(x) + at));
      } else {   // FP8 row with 1x128 scales: the forward's value, rounded once to FP32
        const uint8_t code = static_cast<const uint8_t*>(x)[at];
        __half_raw hr = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
        v = __half2float(__half(hr)) * __ldg(xs + static_cast<size_t>(first + t) * (ld / 128) + cb);
      }
    }
    tile[t * 129 + c] = v;
  }
  __syncthreads();
  float amax = 0.0f;
  for (int t = 0; t < 128; ++t) amax = fmaxf(amax, fabsf(tile[t * 129 + c]));
  if (KIND == 2) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane_id() == 0) red[c >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  }
  const float sc = tile_scale(amax);
  // group-major output: group g is the contiguous matrix [cols][Kg] at
  // cols * d0, so that one GEMM reads it with its own row stride
  uint8_t* qrow = q + static_cast<size_t>(cols) * d0 + static_cast<size_t>(cb * 128 + c) * Kg + (p * 128 - d0);
  for (int t = 0; t < 128; t += 4) {
    const uint32_t w = e4m3x2(__fdiv_rn(tile[t * 129 + c], sc), __fdiv_rn(tile[(t + 1) * 129 + c], sc)) |
                       (e4m3x2(__fdiv_rn(tile[(t + 2) * 129 + c], sc), __fdiv_rn(tile[(t + 3) * 129 + c], sc)) << 16);
    *reinterpret_cast<uint32_t*>(qrow + t) = w;
  }
  const int pg = p - d0 / 128;              // token block within the group
  if (KIND != 2) s[static_cast<size_t>(cols) * (d0 / 128) + static_cast<size_t>(cb * 128 + c) * (Kg / 128) + pg] = sc;
  else if (c == 0) s[static_cast<size_t>(cols / 128) * (d0 / 128) + static_cast<size_t>(cb) * (Kg / 128) + pg] = sc;
}

// dst[b][j][dst_col + i] = src[b][i][j], 32 x 32 tiles through shared memory.
template <typename E>
__global__ void __launch_bounds__(256) transpose_kernel(const E* __restrict__ src, int rows, int cols,
                                                        long long src_bstride, E* __restrict__ dst, int dst_ld,
                                                        int dst_col, long long dst_bstride) {
  __shared__ E t[32][33];
  const int b = blockIdx.z;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const E* sp = src + b * src_bstride;
  E* dp = dst + b * dst_bstride;
  for (int k = threadIdx.y; k < 32; k += 8) {
    const int i = i0 + k, j = j0 + threadIdx.x;
    if (i < rows && j < cols) t[k][threadIdx.x] = sp[static_cast<size_t>(i) * cols + j];
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += 8) {
    const int j = j0 + k, i = i0 + threadIdx.x;
    if (i < rows && j < cols) dp[static_cast<size_t>(j) * dst_ld + dst_col + i] = t[threadIdx.x][k];
  }
}

}  // namespace bwd
}  // namespace moe

extern "C" int moe_swiglu_backward_quant(const float* g, const float* u, const float* dh, int R, int I, float* dgu,
                                         uint8_t* q, float* qs, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(R >= 0 && I > 0);
  MOE_CHECK_SUPPORTED(I % 128 == 0);
  if (R == 0) return MOE_OK;
  MOE_CHECK_ARG(g && u && dh && q && qs);
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(g) % 16 == 0 && reinterpret_cast<uintptr_t>(u) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(dh) % 16 == 0 && reinterpret_cast<uintptr_t>(dgu) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(q) % 4 == 0);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  long long blocks = (static_cast<long long>(R) * (I / 128) + 7) / 8;
  const long long cap = static_cast<long long>(di.sm_count) * 16;
  if (blocks > cap) blocks = cap;
  bwd::swiglu_backward_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(g, u, dh, R, I, dgu, q,
                                                                                              qs);
  return launch_status("moe_swiglu_backward_quant");
}

// kind: 0 FP32 rows, 1 BF16 rows (1x128 tiles along the tokens), 2 FP8 rows with
// 1x128 scales xs (128x128 blocks)
static int quant_t(int kind, const void* x, const float* xs, int ld, int cols, const int32_t* src_off,
                   const int32_t* dst_off, int n_groups, int Ktot, uint8_t* q, float* s, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(ld >= cols && cols > 0 && n_groups >= 1 && Ktot >= 0);
  MOE_CHECK_SUPPORTED(cols % 128 == 0 && Ktot % 128 == 0 && (kind != 2 || ld % 128 == 0));
  if (Ktot == 0) return MOE_OK;
  MOE_CHECK_ARG(x && src_off && dst_off && q && s && (kind != 2 || xs));
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  const size_t sh = 128 * 129 * sizeof(float);
  dim3 grid(Ktot / 128, cols / 128);
  cudaStream_t st = as_stream(stream);
  auto launch = [&](auto kern) -> int {
    if (int e = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sh)),
                            "quant_t smem attribute"))
      return e;
    kern<<<grid, 128, sh, st>>>(x, xs, ld, cols, src_off, dst_off, n_groups, Ktot, q, s);
    return launch_status("transposed quantisation");
  };
  if (kind == 0) return launch(bwd::quant_t_kernel<0>);
  if (kind == 1) return launch(bwd::quant_t_kernel<1>);
  return launch(bwd::quant_t_kernel<2>);
}

extern "C" int moe_quant_1x128_t(const void* x, int x_is_bf16, int ld, int cols, const int32_t* src_off,
                                 const int32_t* dst_off, int n_groups, int Ktot, uint8_t* q, float* s, void* stream) {
  return quant_t(x_is_bf16 ? 1 : 0, x, nullptr, ld, cols, src_off, dst_off, n_groups, Ktot, q, s, stream);
}

extern "C" int moe_quant_128x128_t(const uint8_t* xq, const float* xs, int ld, int cols, const int32_t* src_off,
                                   const int32_t* dst_off, int n_groups, int Ktot, uint8_t* q, float* s,
                                   void* stream) {
  return quant_t(2, xq, xs, ld, cols, src_off, dst_off, n_groups, Ktot, q, s, stream);
}

extern "C" int moe_transpose(const void* src, int elem_bytes, int batch, int rows, int cols, void* dst, int dst_ld,
                             int dst_col, void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(batch >= 0 && rows >= 0 && cols >= 0 && dst_col >= 0 && dst_ld >= dst_col + rows);
  MOE_CHECK_SUPPORTED(elem_bytes == 1 || elem_bytes == 4);
  if (batch == 0 || rows == 0 || cols == 0) return MOE_OK;
  MOE_CHECK_ARG(src && dst);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  MOE_CHECK_SUPPORTED(batch <= 65535);
  dim3 grid((cols + 31) / 32, (rows + 31) / 32, batch), block(32, 8);
  const long long sb = static_cast<long long>(rows) * cols, db = static_cast<long long>(cols) * dst_ld;
  if (elem_bytes == 1)
    bwd::transpose_kernel<uint8_t><<<grid, block, 0, as_stream(stream)>>>(
        static_cast<const uint8_t*>(src), rows, cols, sb, static_cast<uint8_t*>(dst), dst_ld, dst_col, db);
  else
    bwd::transpose_kernel<float><<<grid, block, 0, as_stream(stream)>>>(
        static_cast<const float*>(src), rows, cols, sb, static_cast<float*>(dst), dst_ld, dst_col, db);
  return launch_status("moe_transpose");
}
