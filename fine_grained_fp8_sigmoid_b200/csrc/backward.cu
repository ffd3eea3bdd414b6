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

// One block of 256 threads per (128 tokens, 128 columns). The tile is read
// with 16-byte loads (thread t: token t/2, half t%2 of the columns) and
// staged in shared memory as [token][column] in the input's own type (so
// that several blocks fit an SM); thread t then owns column t%128 over tokens
// (t/128)*64..+64: those values belong to one 1x128 tile of the transposed
// tensor (KIND 0: FP32 input, KIND 1: BF16 input; a scale per column and
// token block, the two halves' max-abs combined) or to one 128x128 block
// (KIND 2: FP8 input with 1x128 scales, each value dequantised and rounded
// once to FP32; one scale for the whole tile). The codes are staged again as
// [column][token] rows and leave as 128-byte row segments.
template <int KIND> struct QtStage;
template <> struct QtStage<0> { using E = float;    static constexpr int LD = 132; };  // elements per row
template <> struct QtStage<1> { using E = uint16_t; static constexpr int LD = 136; };
template <> struct QtStage<2> { using E = uint8_t;  static constexpr int LD = 144; };
constexpr int QT_OUT_LD = 144;    // bytes per staged output row (16-byte aligned, spreads the banks)

template <int KIND>
constexpr size_t qt_smem_bytes() {
  return 128 * QtStage<KIND>::LD * sizeof(typename QtStage<KIND>::E) + 128 * QT_OUT_LD;
}

template <int KIND>
__device__ __forceinline__ float qt_value(const typename QtStage<KIND>::E v, float sx) {
  if (KIND == 0) return v;
  if (KIND == 1) return bf16_bits_to_float(v);
  __half_raw hr = __nv_cvt_fp8_to_halfraw(v, __NV_E4M3);
  return __half2float(__half(hr)) * sx;
}

template <int KIND>
__global__ void __launch_bounds__(256) quant_t_kernel(const void* __restrict__ x, const float* __restrict__ xs,
                                                      int ld, int cols, const int32_t* __restrict__ src_off,
                                                      const int32_t* __restrict__ dst_off, int n_groups, int Ktot,
                                                      uint8_t* __restrict__ q, float* __restrict__ s) {
  using E = typename QtStage<KIND>::E;
  constexpr int LD = QtStage<KIND>::LD;
  constexpr int VEC = 16 / sizeof(E);                 // elements per 16-byte load
  extern __shared__ __align__(16) uint8_t qt_raw[];
  E* tile = reinterpret_cast<E*>(qt_raw);             // [128][LD]
  uint8_t* out = qt_raw + 128 * LD * sizeof(E);       // [128][QT_OUT_LD]
  __shared__ float red[2][128];
  __shared__ float bred[8];
  __shared__ float rsx[128];                          // KIND 2: each token row's 1x128 scale
  const int p = blockIdx.x;                           // token block of the output's K
  const int cb = blockIdx.y;                          // column block
  const int g = block_group(dst_off, n_groups, p * 128);
  const int d0 = __ldg(dst_off + g);
  const int first = __ldg(src_off + g) + (p * 128 - d0);
  const int live = max(0, min(128, __ldg(src_off + g + 1) - first));
  const int tid = threadIdx.x;
  {
    const int r = tid >> 1, h = tid & 1;
    uint4* trow = reinterpret_cast<uint4*>(tile + r * LD + h * 64);
    constexpr int NV = 64 / VEC;
    if (r < live) {
      const size_t at = static_cast<size_t>(first + r) * ld + cb * 128 + h * 64;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const E*>(x) + at);
      uint4 v[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) v[i] = __ldg(src + i);
#pragma unroll
      for (int i = 0; i < NV; ++i) trow[i] = v[i];
      if (KIND == 2 && h == 0) rsx[r] = __ldg(xs + static_cast<size_t>(first + r) * (ld / 128) + cb);
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i) trow[i] = make_uint4(0, 0, 0, 0);
      if (KIND == 2 && h == 0) rsx[r] = 0.0f;
    }
  }
  __syncthreads();
  const int c = tid & 127, th = tid >> 7;
  const E* tcol = tile + th * 64 * LD + c;
  const float* sxc = rsx + th * 64;
  float amax = 0.0f;
#pragma unroll 8
  for (int t = 0; t < 64; ++t) amax = fmaxf(amax, fabsf(qt_value<KIND>(tcol[t * LD], KIND == 2 ? sxc[t] : 0.0f)));
  if (KIND != 2) {
    red[th][c] = amax;
    __syncthreads();
    amax = fmaxf(red[0][c], red[1][c]);
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane_id() == 0) bred[tid >> 5] = amax;
    __syncthreads();
    amax = bred[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, bred[i]);
  }
  const float sc = tile_scale(amax);
  uint8_t* orow = out + c * QT_OUT_LD + th * 64;
#pragma unroll
  for (int t = 0; t < 64; t += 16) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tt = t + 4 * k + e;
        v[e] = __fdiv_rn(qt_value<KIND>(tcol[tt * LD], KIND == 2 ? sxc[tt] : 0.0f), sc);
      }
      w[k] = e4m3x2(v[0], v[1]) | (e4m3x2(v[2], v[3]) << 16);
    }
    *reinterpret_cast<uint4*>(orow + t) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (KIND != 2) {
    if (th == 0) s[static_cast<size_t>(cb * 128 + c) * (Ktot / 128) + p] = sc;
  } else if (tid == 0) {
    s[static_cast<size_t>(cb) * (Ktot / 128) + p] = sc;
  }
  __syncthreads();
  // output [cols][Ktot]: group g holds columns d0 .. d0 + K_g of every row,
  // so one K-grouped GEMM reads all groups through one tensor map; eight
  // threads write one row's 128 bytes of this token block
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int row = pass * 32 + (tid >> 3), chunk = tid & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(out + row * QT_OUT_LD + chunk * 16);
    *reinterpret_cast<uint4*>(q + static_cast<size_t>(cb * 128 + row) * Ktot + static_cast<size_t>(p) * 128 +
                              chunk * 16) = v;
  }
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
  const size_t esz = kind == 0 ? 4 : kind == 1 ? 2 : 1;
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(x) % 16 == 0 && (static_cast<size_t>(ld) * esz) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(q) % 16 == 0);
  dim3 grid(Ktot / 128, cols / 128);
  cudaStream_t st = as_stream(stream);
  auto launch = [&](auto kern, size_t sh) -> int {
    if (int e = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sh)),
                            "quant_t smem attribute"))
      return e;
    kern<<<grid, 256, sh, st>>>(x, xs, ld, cols, src_off, dst_off, n_groups, Ktot, q, s);
    return launch_status("transposed quantisation");
  };
  if (kind == 0) return launch(bwd::quant_t_kernel<0>, bwd::qt_smem_bytes<0>());
  if (kind == 1) return launch(bwd::quant_t_kernel<1>, bwd::qt_smem_bytes<1>());
  return launch(bwd::quant_t_kernel<2>, bwd::qt_smem_bytes<2>());
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
