// Router: s_{i,t} = Sigmoid(u_t . e_i), biased top-K_r selection, normalised
// gates ("DeepSeek-V3 Teknik Raporu", Yöntem 2; "DeepSeek-V3 Technical
// Report" (fr), Méthode 2).
//
// The logits are a [T x d] x [d x N_r] product on the tensor cores. One CTA
// takes 128 tokens and all experts (the MMA is N = 256; experts beyond N_r
// read zero rows). u and e stream through shared memory with TMA in 128-byte
// swizzled K blocks of 64 bf16. Each K block's four tcgen05 kind::f16 MMAs
// (BF16 x BF16 -> FP32) write a fresh TMEM partial, and the epilogue warps add
// the partials in FP32 registers. Accumulating all of d = 7168 inside the
// tensor core lets its truncating accumulation drift by ~1e-4 in the logit;
// each TMEM partial here covers RK = 4 K blocks (256 channels) and the
// epilogue adds the partials in FP32 registers, which keeps the error near
// FP32 rounding while reading the 128 x 256 partial back only every fourth
// K block (the read-back competes with the MMAs for TMEM).
// After the K loop the logits are parked in the (now idle) pipeline shared
// memory as [expert][token].
//
// Split K: with few token tiles (decode: one), a single CTA per tile would
// stream all of d through one SM. The launch then forms clusters of S CTAs
// per tile (S a power of two <= 8, S * tiles <= SMs); CTA rank r of the
// cluster runs its share of the K groups and parks its FP32 partial logits.
// After a cluster barrier every rank takes 128/S of the tile's tokens: a
// token's experts are spread over 2S threads of consecutive lanes, each adds
// the ranks' partials in rank order through distributed shared memory
// (deterministic), forms the affinity and biased key and keeps a top-K list,
// and the 2S lists merge by shuffles. A second cluster barrier keeps every
// rank's shared memory alive until all ranks have read it.
// Warp roles (384 threads): warp 0 TMA, warp 1 MMA + TMEM, warps 4-11
// epilogue (TMEM lane quadrant w%4, column half (w-4)/4 while reading TMEM).
//
// Fused activation quantisation (xq non-null): the u tiles that stream
// through shared memory for the logits are also the input of step 5 of the
// layer, E4M3 in 1x128 tiles ("DeepSeek-V3 Teknik Raporu", Temel fikirler,
// FP8 bullet). Two consecutive 64-channel K blocks hold one 1x128 tile per
// token: epilogue thread (token r, half h) reads its token's 64 values of K
// block 2p + h from the stage (otherwise idle during the K loop: the MMAs
// are the logits' critical path), the two halves' max-abs meet through a
// named barrier, and each half writes its 64 codes (half 0 the scale) with
// the same arithmetic as moe_quant_1x128. A stage is refilled only after the
// MMA commit and the four warps that read it have released it.
#include <mutex>

#include "host.cuh"

namespace moe {
namespace route {

constexpr int BM = 128;          // tokens per CTA (TMEM lanes)
constexpr int PR = 260;          // parked logits: floats per token row (256 experts + 4 pad, 16-byte rows)
constexpr int BK = 64;           // bf16 per K block = 128 bytes = one swizzle row
constexpr int NP = 256;          // MMA N: all experts of a token in one tile
constexpr int STAGES = 4;
constexpr int RK = 4;            // K blocks per TMEM partial
constexpr int THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int EPI_THREADS = 256;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = NP * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * NP;
constexpr uint32_t REGS_CTRL = 56;
constexpr uint32_t REGS_EPI = 224;

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

// sigmoid with the hardware exponential and approximate division (relative
// error ~1e-6, far inside the routing acceptance margin); sigmoid(0) = 0.5
// exactly, and the limits 0 (z -> -inf: 1 / inf) and 1 hold
__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }

// top-K of (key, index) pairs, keys descending; strict comparison, so an
// equal key inserted later (a higher index) stays behind
template <int KMAX>
__device__ __forceinline__ void topk_insert_ki(float (&kk)[KMAX], int (&ii)[KMAX], float key, int idx) {
  bool shifting = false;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const bool take = shifting || (key > kk[j]);
    const float tk = kk[j];
    const int ti = ii[j];
    kk[j] = take ? key : tk;
    ii[j] = take ? idx : ti;
    key = take ? tk : key;
    idx = take ? ti : idx;
    shifting = take;
  }
}

template <int KMAX>
struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float bias[NP];
  float qamax[2][2][BM];      // fused quantisation: [pair parity][half][token] max-abs
};

static_assert(BM * PR * 4 <= STAGES * STAGE_BYTES, "parked logits fit the pipeline stages");

template <int KMAX>
constexpr size_t router_smem_bytes() {
  return 1024 + STAGES * STAGE_BYTES + sizeof(Smem<KMAX>);
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// FP32 at byte offset `off` from `base` (a shared-memory address of this
// CTA) in CTA `rank` of the cluster
__device__ __forceinline__ float ld_cluster_f32(uint32_t base, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(base), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Two float4 at base + off0 and base + off1 in CTA `rank` of the cluster
__device__ __forceinline__ void ld_cluster_f32x4x2(uint32_t base, uint32_t off0, uint32_t off1, uint32_t rank,
                                                   float (&v)[8]) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(base), "r"(rank));
  asm volatile(
      "ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%8];\n\t"
      "ld.shared::cluster.v4.f32 {%4, %5, %6, %7}, [%9];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
      : "r"(remote + off0), "r"(remote + off1)
      : "memory");
}

// Merges one (key, index) into a top-K list ordered by key descending, then
// index ascending, whatever the order the entries arrive in.
template <int KMAX>
__device__ __forceinline__ void topk_insert_lex(float (&kk)[KMAX], int (&ii)[KMAX], float key, int idx) {
  bool shifting = false;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const bool take = shifting || key > kk[j] || (key == kk[j] && idx < ii[j]);
    const float tk = kk[j];
    const int ti = ii[j];
    kk[j] = take ? key : tk;
    ii[j] = take ? idx : ti;
    key = take ? tk : key;
    idx = take ? ti : idx;
    shifting = take;
  }
}

// Named barrier over n threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Eight bf16 of a 16-byte chunk as floats.
__device__ __forceinline__ void bf16x8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFF);
    f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}

template <int KMAX>
__global__ void __launch_bounds__(THREADS, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_e,
                  const float* __restrict__ b, int T, int d, int N_r, int K, int S,
                  float* __restrict__ scores_out, int32_t* __restrict__ topk_idx,
                  float* __restrict__ gates, uint8_t* __restrict__ xq, float* __restrict__ xs) {
  extern __shared__ uint8_t smem_raw[];
  // operand tiles need 1024-byte alignment for the 128-byte swizzle
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem<KMAX>& sm = *reinterpret_cast<Smem<KMAX>*>(tiles + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int tile = blockIdx.x / S;
  const int rank = blockIdx.x % S;          // rank in the cluster of S CTAs (1-D clusters)
  const int KB = d / BK;
  // this rank's K blocks: whole partial groups of RK blocks
  const int NG_all = (KB + RK - 1) / RK;
  const int g_lo = rank * NG_all / S, g_hi = (rank + 1) * NG_all / S;
  const int kb_lo = g_lo * RK, kb_hi = min(g_hi * RK, KB);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      // the MMA commit, and with the fused quantisation the four epilogue
      // warps that read the stage's u rows
      mbar_init(&sm.empty[s], xq != nullptr ? 1 + 4 : 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.tfull[i], 1);
      mbar_init(&sm.tempty[i], EPI_THREADS / 32);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_u);
    tma_prefetch_desc(&tm_e);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < NP; i += THREADS) sm.bias[i] = i < N_r ? b[i] : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp < EPI_WARP0) {
    regs_decrease<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // producer: K blocks of u (128 x 64) and e (256 x 64, rows >= N_r read as zero)
      int armed[STAGES];
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        const int s = (kb - kb_lo) % STAGES;
        const uint32_t ph = ((kb - kb_lo) / STAGES) & 1;
        if (!mbar_wait(&sm.empty[s], ph ^ 1, abort)) break;
        uint8_t* a_dst = tiles + s * STAGE_BYTES;
        mbar_arrive_expect_tx(&sm.full[s], STAGE_BYTES);
        tma_load_2d(a_dst, &tm_u, &sm.full[s], kb * BK, tile * BM);
        tma_load_2d(a_dst + A_BYTES, &tm_e, &sm.full[s], kb * BK, 0);
        armed[s] = ph;
      }
      if (*abort) {
        // let every issued copy land before the block's shared memory is released
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (armed[s] >= 0) mbar_wait(&sm.full[s], armed[s], &never, 100000000ull);
      }
    } else if (warp == 1 && lane == 0) {
      const uint32_t idesc = make_idesc(1, 1, BM, NP);
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        const int s = (kb - kb_lo) % STAGES;
        const uint32_t ph = ((kb - kb_lo) / STAGES) & 1;
        const int grp = kb / RK - g_lo;          // partial buffer group of this rank
        const int buf = grp & 1;
        const bool first = kb % RK == 0, last = kb % RK == RK - 1 || kb == KB - 1;
        if (first && !mbar_wait(&sm.tempty[buf], ((grp >> 1) & 1) ^ 1, abort)) break;
        if (!mbar_wait(&sm.full[s], ph, abort)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + s * STAGE_BYTES);
        const uint64_t ad = sw128_kmajor_desc(a_addr);
        const uint64_t bd = sw128_kmajor_desc(a_addr + A_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)  // 16 bf16 = 32 bytes per MMA
          umma_f16(tmem + buf * NP, ad + 2 * k, bd + 2 * k, idesc, (k != 0) || !first);
        umma_commit(&sm.empty[s]);
        if (last) umma_commit(&sm.tfull[buf]);
      }
      // all MMAs of this thread complete before TMEM is released
      umma_commit(&sm.drain);
      volatile int never = 0;
      mbar_wait(&sm.drain, 0, &never, 100000000ull);
    }
  } else {
    regs_increase<REGS_EPI>();
    const int q = warp & 3;
    const int half = (warp - EPI_WARP0) >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    float acc[128];
#pragma unroll
    for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
    bool ok = true;
    const int NG = g_hi - g_lo;
    int qpar = 0;
    for (int grp = 0; grp < NG; ++grp) {
      if (xq != nullptr) {
        // quantise the 1x128 tiles of this partial group's K blocks
        const int kb_a = kb_lo + grp * RK, kb_b = min(kb_a + RK, kb_hi);
        for (int kb0 = kb_a; kb0 < kb_b; kb0 += 2) {
          const int kb = kb0 + half;
          const int st = (kb - kb_lo) % STAGES;
          const bool okw = warp_wait(&sm.full[st], ((kb - kb_lo) / STAGES) & 1, abort);
          const uint8_t* urow = tiles + st * STAGE_BYTES + r * 128;   // 128-byte swizzled row r
          float amax = 0.0f;
          if (okw) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float f[8];
              bf16x8(*reinterpret_cast<const uint4*>(urow + ((c ^ (r & 7)) << 4)), f);
#pragma unroll
              for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            }
          }
          sm.qamax[qpar][half][r] = amax;
          if (named_bar_or(2, EPI_THREADS, !okw || *abort)) { ok = false; break; }
          amax = fmaxf(amax, sm.qamax[qpar][half ^ 1][r]);
          qpar ^= 1;
          const float sc = tile_scale(amax);
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float f[8];
            bf16x8(*reinterpret_cast<const uint4*>(urow + ((c ^ (r & 7)) << 4)), f);
            w[2 * c] = e4m3x2(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc)) |
                       (e4m3x2(__fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc)) << 16);
            w[2 * c + 1] = e4m3x2(__fdiv_rn(f[4], sc), __fdiv_rn(f[5], sc)) |
                           (e4m3x2(__fdiv_rn(f[6], sc), __fdiv_rn(f[7], sc)) << 16);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.empty[st]);     // this warp is done with the stage
          const int tok = tile * BM + r;
          if (tok < T) {
            uint4* dst = reinterpret_cast<uint4*>(xq + static_cast<size_t>(tok) * d + kb * BK);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
            if (half == 0) xs[static_cast<size_t>(tok) * (d / 128) + kb0 / 2] = sc;
          }
        }
        if (!ok) break;
      }
      const int buf = grp & 1;
      const bool okt = warp_wait(&sm.tfull[buf], (grp >> 1) & 1, abort);
      // with the fused quantisation every epilogue warp must leave the loop
      // together (its barriers count all of them)
      if (xq != nullptr ? named_bar_or(2, EPI_THREADS, !okt) : !okt) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + buf * NP + half * 128 + c * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[c * 32 + j] += v[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tempty[buf]);
    }
    // Every TMA load was consumed by an MMA and every MMA has completed (the
    // last partial has been read), so the stage buffers are free: park this
    // CTA's partial logits there as [token][expert] rows of PR floats
    // (16-byte stores; readers take 16-byte runs of a token's row).
    float* park = reinterpret_cast<float*>(tiles);
    if (ok) {
      float4* row = reinterpret_cast<float4*>(park + r * PR + half * 128);
#pragma unroll
      for (int m = 0; m < 32; ++m) row[m] = make_float4(acc[4 * m], acc[4 * m + 1], acc[4 * m + 2], acc[4 * m + 3]);
    }
    if (S > 1) cluster_sync_all();           // every rank's partial is parked
    else named_bar_sync(1, EPI_THREADS);

    // The tile's tokens are split over the S ranks, a token's experts over
    // TPT = 2S threads in consecutive lanes: thread ch owns the runs of 4
    // experts 4*(ch + TPT*m), so a warp's 16-byte loads of a token's row are
    // contiguous. A thread adds the ranks' partials in rank order, forms the
    // affinity and the biased key, and keeps a top-K list; the TPT lists of a
    // token then merge in a butterfly of shuffles.
    const int TPC = BM / S, TPT = EPI_THREADS / TPC, RUNS = NP / (4 * TPT);
    const int etid = (warp - EPI_WARP0) * 32 + lane;
    const int rr = rank * TPC + etid / TPT;     // token row in the tile
    const int ch = etid % TPT;
    const int tt = tile * BM + rr;
    float* srow = (scores_out != nullptr && tt < T) ? scores_out + static_cast<size_t>(tt) * N_r : nullptr;
    const uint32_t tok_base = smem_u32(park + rr * PR);   // this token's row, this CTA
    // two insertion lists (the two runs of each step), merged at the end
    float ka[KMAX], kb2[KMAX];
    int ia[KMAX], ib[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ka[j] = kb2[j] = -INFINITY;
      ia[j] = ib[j] = 0x7fffffff;
    }
#pragma unroll 1
    for (int m = 0; m < RUNS; m += 2) {        // RUNS = 32 / S: 4 (S = 8) .. 32 (S = 1)
      const int ca = 4 * (ch + TPT * m), cb = 4 * (ch + TPT * (m + 1));
      if (ca >= N_r) break;                    // every later run starts higher
      float z[8];
      if (S == 1) {
        const float4 a0 = *reinterpret_cast<const float4*>(park + rr * PR + ca);
        const float4 a1 = *reinterpret_cast<const float4*>(park + rr * PR + cb);
        z[0] = a0.x; z[1] = a0.y; z[2] = a0.z; z[3] = a0.w;
        z[4] = a1.x; z[5] = a1.y; z[6] = a1.z; z[7] = a1.w;
      } else {
        // every rank's values in flight before the sums (in rank order)
        float v[8][8];
#pragma unroll
        for (int q2 = 0; q2 < 8; ++q2)
          if (q2 < S) ld_cluster_f32x4x2(tok_base, ca * 4, cb * 4, q2, v[q2]);
#pragma unroll
        for (int k = 0; k < 8; ++k) z[k] = v[0][k];
#pragma unroll
        for (int q2 = 1; q2 < 8; ++q2)
          if (q2 < S)
#pragma unroll
            for (int k = 0; k < 8; ++k) z[k] += v[q2][k];
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int c = (k < 4 ? ca : cb) + (k & 3);
        if (c < N_r) {
          const float sg = sigmoid_fast(z[k]);
          if (k < 4) topk_insert_ki(ka, ia, sg + sm.bias[c], c);
          else topk_insert_ki(kb2, ib, sg + sm.bias[c], c);
          if (srow != nullptr) srow[c] = sg;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (ib[j] < N_r) topk_insert_lex(ka, ia, kb2[j], ib[j]);
    for (int m = 1; m < TPT; m <<= 1) {
      float pk[KMAX];
      int pi[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        pk[j] = __shfl_xor_sync(0xffffffffu, ka[j], m);
        pi[j] = __shfl_xor_sync(0xffffffffu, ia[j], m);
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (pi[j] < N_r) topk_insert_lex(ka, ia, pk[j], pi[j]);
    }
    if (ch == 0 && tt < T) {
      // the affinities of the selected experts, from the same summed logits
      float ss[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        float zz = 0.0f;
        if (ia[j] < N_r) {
          const uint32_t o = static_cast<uint32_t>(ia[j]) * 4;
          if (S == 1) zz = park[rr * PR + ia[j]];
          else
            for (int q2 = 0; q2 < S; ++q2) zz += ld_cluster_f32(tok_base + o, q2);
        }
        ss[j] = ia[j] < N_r ? sigmoid_fast(zz) : 0.0f;
      }
      topk_store(ia, ss, K, topk_idx + static_cast<size_t>(tt) * K, gates + static_cast<size_t>(tt) * K);
    }
  }
  if (S > 1) {
    // the control warps meet the epilogue's first barrier here; the second
    // keeps every rank's parked partial alive until rank 0 has read it
    __syncwarp();
    if (warp < EPI_WARP0) cluster_sync_all();
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
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

static int route_launch(const uint16_t* u, const uint16_t* e, const float* b, const float* scores_in, int T, int d,
                        int N_r, int K_r, float* scores_out, int32_t* topk_idx, float* gates, uint8_t* xq, float* xs,
                        void* stream) {
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
  CUtensorMap tm_u, tm_e;
  if (int st = make_tmap_2d(&tm_u, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, d, BM, BK)) return st;
  if (int st = make_tmap_2d(&tm_e, e, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N_r, d, NP, BK)) return st;
  const int tiles = (T + BM - 1) / BM;
  const int NG_all = (d / BK + RK - 1) / RK;
  auto k = K_r <= 8 ? router_kernel<8> : router_kernel<16>;
  const size_t smem = K_r <= 8 ? router_smem_bytes<8>() : router_smem_bytes<16>();
  if (int st = cuda_status(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                           "router smem attribute"))
    return st;
  // split K over a cluster of S CTAs per token tile while the SMs allow, up
  // to the largest cluster the device can place (queried once per device and
  // kernel variant)
  static std::mutex mu;
  static int max_cluster[64][2] = {};
  int dev = 0;
  if (int st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice")) return st;
  if (dev < 0 || dev >= 64) return MOE_ERR_NO_DEVICE;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  const int variant = K_r <= 8 ? 0 : 1;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (max_cluster[dev][variant] == 0) {
      int m = 8;
      for (; m > 1; m /= 2) {
        cfg.gridDim = dim3(m);
        attr[0].val.clusterDim.x = m;
        int n_clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&n_clusters, k, &cfg) == cudaSuccess && n_clusters > 0) break;
        cudaGetLastError();
      }
      max_cluster[dev][variant] = m;
    }
  }
  int S = 1;
  while (S < max_cluster[dev][variant] && tiles * S * 2 <= di.sm_count && S * 2 <= NG_all) S *= 2;
  cfg.gridDim = dim3(tiles * S);
  attr[0].val.clusterDim.x = S;
  if (int st = cuda_status(cudaLaunchKernelEx(&cfg, k, tm_u, tm_e, b, T, d, N_r, K_r, S, scores_out, topk_idx, gates,
                                              xq, xs),
                           "router launch"))
    return st;
  return launch_status();
}

extern "C" int moe_route(const uint16_t* u, const uint16_t* e, const float* b, const float* scores_in, int T, int d,
                         int N_r, int K_r, float* scores_out, int32_t* topk_idx, float* gates, void* stream) {
  return route_launch(u, e, b, scores_in, T, d, N_r, K_r, scores_out, topk_idx, gates, nullptr, nullptr, stream);
}

extern "C" int moe_route_quant(const uint16_t* u, const uint16_t* e, const float* b, int T, int d, int N_r, int K_r,
                               float* scores_out, int32_t* topk_idx, float* gates, uint8_t* xq, float* xs,
                               void* stream) {
  using namespace moe;
  MOE_CHECK_ARG(T >= 0 && d >= 0);
  MOE_CHECK_SUPPORTED(d % 128 == 0);
  if (T > 0) {
    MOE_CHECK_ARG(u && xq && xs);
    MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(xq) % 16 == 0);
  }
  return route_launch(u, e, b, nullptr, T, d, N_r, K_r, scores_out, topk_idx, gates, xq, xs, stream);
}
