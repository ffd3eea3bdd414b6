// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory, with its scratch in a fixed array compiled into the library.
//
// Some callers hold only their own input and output buffers and may not
// allocate: an inference engine's plugin whose execute step is forbidden to
// allocate and reserved no workspace for this layer, or a serving loop that
// runs inside a fixed memory budget where cudaMalloc could also stall the
// device. They call this entry point instead of moe_permute; it runs the same
// kernels on a scratch table that lives in g_permute_scratch below.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kStaticScratchBytes of it until the process exits. Its name in
// host code is only a host-side stand-in: the device address is looked up
// with cudaGetSymbolAddress, once per device, with that device current, on
// the first call made on that device.
#include "host.cuh"

namespace moe {
namespace perm {

// 1 MiB: holds the two int32 tables of ceil(T/256) x N_r for, e.g., up to
// 131072 tokens with 256 experts or 32768 tokens with 1024 experts.
constexpr size_t kStaticScratchBytes = size_t(1) << 20;

static __device__ __align__(256) int32_t g_permute_scratch[kStaticScratchBytes / sizeof(int32_t)];

// Device address of g_permute_scratch on the current device; looked up on the
// first call per device and cached.
static int static_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (int st = cuda_status(cudaGetDevice(&dev), "moe_permute_noalloc: cudaGetDevice")) return st;
  if (dev < 0 || dev >= 64) return record_failure(MOE_ERR_NO_DEVICE, "moe_permute_noalloc", "device index out of range");
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (int st = cuda_status(cudaGetSymbolAddress(&p, g_permute_scratch),
                             "moe_permute_noalloc: cudaGetSymbolAddress"))
      return st;
    addr[dev] = p;
  }
  *out = addr[dev];
  return MOE_OK;
}

}  // namespace perm
}  // namespace moe

extern "C" int moe_permute_noalloc(const int32_t* topk_idx, int T, int K_r, int N_r, const uint8_t* xq,
                                   const float* xs, int d, int32_t* counts, int32_t* offsets,
                                   int32_t* sorted_token, int32_t* inv, uint8_t* xq_perm, float* xs_perm,
                                   void* stream) {
  using namespace moe;
  using namespace moe::perm;
  MOE_CHECK_ARG(T >= 0 && K_r >= 1 && N_r >= 1);
  const size_t need = moe_permute_workspace(T, N_r);
  if (need > kStaticScratchBytes) {
    char what[160];
    snprintf(what, sizeof what,
             "T=%d, N_r=%d need %zu bytes of scratch; the static buffer holds %zu (use moe_permute)", T, N_r,
             need, kStaticScratchBytes);
    return record_failure(MOE_ERR_UNSUPPORTED, "moe_permute_noalloc", what);
  }
  void* scratch = nullptr;
  if (int st = static_scratch_address(&scratch)) return st;
  // Every entry of the two tables that a call reads is first written by the
  // same call, so nothing has to be cleared between calls.
  return moe_permute(topk_idx, T, K_r, N_r, xq, xs, d, counts, offsets, sorted_token, inv, xq_perm, xs_perm,
                     scratch, kStaticScratchBytes, stream);
}
