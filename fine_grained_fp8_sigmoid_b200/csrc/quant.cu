// E4M3 quantisers: 1x128 tiles for activations, 128x128 blocks for weights
// ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8 bullet). Scale rule:
// scale = fl32(amax / 448) (1 if zero), q = E4M3_RNE_satfinite(fl32(x / scale)).
#include "host.cuh"

namespace moe {

// Half a warp per 1x128 tile: each lane holds 8 consecutive bf16 (16 bytes),
// so a warp reads 512 contiguous bytes (two tiles) per step and writes 256
// bytes of codes; the max-abs is reduced over the 16 lanes of a tile.
__global__ void __launch_bounds__(256) quant_1x128_kernel(const uint16_t* __restrict__ x,
                                                          long long n_tiles, int tiles_per_row,
                                                          uint8_t* __restrict__ q,
                                                          float* __restrict__ scale) {
  const int lane = lane_id();
  const int sub = lane & 15;                 // lane within the tile
  const long long n_pairs = (n_tiles + 1) / 2;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long pr = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); pr < n_pairs; pr += warps) {
    const long long tile = pr * 2 + (lane >> 4);
    const bool live = tile < n_tiles;         // the last pair may hold one tile
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (live) raw = __ldg(reinterpret_cast<const uint4*>(x + tile * 128) + sub);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_bits_to_float(w[i] & 0xFFFF);
      v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = tile_scale(amax);
    uint32_t c[2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
      c[i] = e4m3x2(__fdiv_rn(v[4 * i], s), __fdiv_rn(v[4 * i + 1], s)) |
             (e4m3x2(__fdiv_rn(v[4 * i + 2], s), __fdiv_rn(v[4 * i + 3], s)) << 16);
    if (live) {
      reinterpret_cast<uint2*>(q + tile * 128)[sub] = make_uint2(c[0], c[1]);
      if (sub == 0) scale[tile] = s;          // tiles are numbered row-major: [row][col/128]
    }
  }
  (void)tiles_per_row;
}

// One block of 256 threads per 128x128 block: thread t owns 64 consecutive
// elements (half a row) and keeps them in registers between the max-abs
// reduction and the conversion.
__global__ void __launch_bounds__(256) quant_128x128_kernel(const float* __restrict__ w,
                                                            int rows, int cols,
                                                            uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  __shared__ float red[8];
  const int bi = blockIdx.y, bj = blockIdx.x;
  const int r = bi * 128 + (threadIdx.x >> 1);
  const int c0 = bj * 128 + (threadIdx.x & 1) * 64;
  const float4* src = reinterpret_cast<const float4*>(w + static_cast<size_t>(r) * cols + c0);
  float4 v[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = __ldg(src + i);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane_id() == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = tile_scale(amax);
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t lo = e4m3x2(__fdiv_rn(v[i].x, s), __fdiv_rn(v[i].y, s));
    const uint32_t hi = e4m3x2(__fdiv_rn(v[i].z, s), __fdiv_rn(v[i].w, s));
    packed[i] = lo | (hi << 16);
  }
  uint4* dst = reinterpret_cast<uint4*>(q + static_cast<size_t>(r) * cols + c0);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  if (threadIdx.x == 0) scale[bi * (cols / 128) + bj] = s;
  (void)rows;
}

}  // namespace moe

extern "C" int moe_quant_1x128(const uint16_t* x, int rows, int cols, uint8_t* q, float* scale,
                               void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(rows >= 0 && cols >= 0);
  MOE_CHECK_SUPPORTED(cols % 128 == 0);
  if (rows == 0 || cols == 0) return MOE_OK;
  MOE_CHECK_ARG(x && q && scale);
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(x) % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 8 == 0);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  const long long n_tiles = static_cast<long long>(rows) * (cols / 128);
  long long blocks = (n_tiles + 15) / 16;   // 8 warps of two tiles each
  const long long cap = static_cast<long long>(di.sm_count) * 16;
  if (blocks > cap) blocks = cap;
  quant_1x128_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      x, n_tiles, cols / 128, q, scale);
  return launch_status();
}

extern "C" int moe_quant_128x128(const float* w, int rows, int cols, uint8_t* q, float* scale,
                                 void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(rows >= 0 && cols >= 0);
  MOE_CHECK_SUPPORTED(rows % 128 == 0 && cols % 128 == 0);
  if (rows == 0 || cols == 0) return MOE_OK;
  MOE_CHECK_ARG(w && q && scale);
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(w) % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 16 == 0);
  MOE_CHECK_SUPPORTED(rows / 128 <= 65535);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  dim3 grid(cols / 128, rows / 128);
  quant_128x128_kernel<<<grid, 256, 0, as_stream(stream)>>>(w, rows, cols, q, scale);
  return launch_status();
}
