// Row movement for expert parallelism: the pieces of the dispatch and the
// return path that are not the layer's arithmetic. The exchanges themselves
// (all-to-all of rows between the GPUs) run in NCCL; these kernels prepare
// and undo the orderings around them.
//
//   moe_group_of_rows - the group (modulo a count) of every row of a grouped
//                       layout, from its offsets: on the receiving GPU, the
//                       local expert of each received row.
//   moe_gather_rows   - dst[i] = src[idx[i]] for rows of any width (a
//                       multiple of 4 bytes): expert outputs back into
//                       arrival order before they return.
#include "host.cuh"

namespace moe {
namespace ep {

__global__ void __launch_bounds__(256) group_of_rows_kernel(const int32_t* __restrict__ offsets, int n_groups,
                                                            int modulo, int n_rows, int32_t* __restrict__ out) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n_rows) return;
  int lo = 0, hi = n_groups - 1;   // last group g with offsets[g] <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= p) lo = mid; else hi = mid - 1;
  }
  out[p] = lo % modulo;
}

// One warp per row, in vectors of V (16-byte or 4-byte words).
template <typename V>
__global__ void __launch_bounds__(256) gather_rows_kernel(const V* __restrict__ src, int n_src,
                                                          const int32_t* __restrict__ idx, int n, int vec_per_row,
                                                          V* __restrict__ dst) {
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long i = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); i < n; i += warps) {
    const int r = __ldg(idx + i);
    if (r < 0 || r >= n_src) {
      if (lane_id() == 0) set_device_error(MOE_ERR_INVALID_ARG);
      continue;
    }
    const V* s = src + static_cast<size_t>(r) * vec_per_row;
    V* d = dst + static_cast<size_t>(i) * vec_per_row;
    for (int v = lane_id(); v < vec_per_row; v += 32) d[v] = __ldg(s + v);
  }
}

}  // namespace ep
}  // namespace moe

extern "C" int moe_group_of_rows(const int32_t* offsets, int n_groups, int modulo, int n_rows, int32_t* out,
                                 void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(n_groups >= 1 && modulo >= 1 && n_rows >= 0);
  if (n_rows == 0) return MOE_OK;
  MOE_CHECK_ARG(offsets && out);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  ep::group_of_rows_kernel<<<(n_rows + 255) / 256, 256, 0, as_stream(stream)>>>(offsets, n_groups, modulo, n_rows,
                                                                                   out);
  return launch_status("moe_group_of_rows");
}

extern "C" int moe_gather_rows(const void* src, int n_src, const int32_t* idx, int n, int row_bytes, void* dst,
                               void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(n_src >= 0 && n >= 0 && row_bytes > 0);
  MOE_CHECK_SUPPORTED(row_bytes % 4 == 0);
  if (n == 0) return MOE_OK;
  MOE_CHECK_ARG(src && idx && dst && n_src > 0);
  const bool wide = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(dst) % 16 == 0;
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(src) % 4 == 0 && reinterpret_cast<uintptr_t>(dst) % 4 == 0);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  long long blocks = (static_cast<long long>(n) + 7) / 8;
  const long long cap = static_cast<long long>(di.sm_count) * 16;
  if (blocks > cap) blocks = cap;
  if (wide)
    ep::gather_rows_kernel<uint4><<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
        static_cast<const uint4*>(src), n_src, idx, n, row_bytes / 16, static_cast<uint4*>(dst));
  else
    ep::gather_rows_kernel<uint32_t><<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
        static_cast<const uint32_t*>(src), n_src, idx, n, row_bytes / 4, static_cast<uint32_t*>(dst));
  return launch_status("moe_gather_rows");
}
