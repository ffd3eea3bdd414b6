// Narrow tiles of the grouped FP8 GEMM: groups (or the last rows of a group)
// with at most 64 tokens.
//
// A 128-row tile of the wide kernel pays a full 128 x 256 x 32 MMA and reads
// back a 128 x 256 FP32 partial per K block however few rows are real. For a
// few tokens the roles are swapped: 128 weight rows are the MMA's M side and
// the tokens its N side (N = rows rounded up to 16, at most 64), so
//     D[c, j] = sum_kb s_W[c/128, kb] * s_X[j, kb] * (W_kb[c] . X_kb[j])
// with the same FP32 promotion per 128-wide K block
// ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8 bullet). An MMA with
// N <= 64 costs a third of an N = 256 one, and each partial holds at most
// 2 x 64 columns, so TMEM keeps four partial buffers instead of two.
//
// A group of r rows is split into floor(r / 128) wide tiles plus, when the
// remainder is 1..64 rows, one narrow tile here (a remainder above 64 stays
// a padded wide tile). Decode batches (a few tokens per expert) run almost
// entirely here.
//
// Tiles (persistent CTA per SM, same roles as the wide kernel):
//   phase 1: (group g, 128 intermediate channels n): MMAs W_gate[n] x X^T and
//            W_up[n] x X^T into columns [0, N) and [64, 64 + N) of a buffer.
//            Epilogue thread = one channel (TMEM lane) x 32 tokens (warps
//            4-7 tokens 0-31, warps 8-11 tokens 32-63); SwiGLU, then the
//            1x128 requantisation of each token's 128 channels, whose
//            max-abs runs across lanes and across the four lane-quadrant
//            warps.
//   phase 2: (group g, 256 output channels n): MMAs W_down[n*256 .. +128] x
//            H^T and W_down[n*256+128 .. +256] x H^T. Epilogue thread = one
//            output channel x all tokens; a warp stores 32 consecutive
//            channels of one token (128 bytes) at a time.

namespace moe {
namespace gn {

using gg::Args;

constexpr int BK = 128;
constexpr int NMAX = 64;                         // tokens per narrow tile
constexpr int WIDE_ROWS = 128;
constexpr int A_BYTES = 128 * BK;                // one 128-row weight tile
constexpr int B_BYTES = NMAX * BK;               // up to 64 token rows
constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
constexpr int STAGES = 4;
constexpr int NBUF = 4;                          // TMEM partial buffers of 128 columns
constexpr int THREADS = 384;
constexpr int EPI_WARPS = 8;
constexpr int EPI_WARP0 = 4;
constexpr uint32_t REGS_CTRL = 56;
constexpr uint32_t REGS_EPI = 224;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_KB = 56;                       // K blocks per tile held in shared memory (d, I <= 7168)

struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[NBUF];
  uint64_t tempty[NBUF];
  uint64_t drain;
  uint64_t sbar;                  // token scales of the tile staged (per tile parity)
  uint64_t xbar;                  // per-token max-abs partials written (phase 1)
  uint32_t tmem_base;
  int abort;
  int total_tiles;
  int tile_start[gg::MAX_GROUPS + 1];
  int off[gg::MAX_GROUPS + 1];
  // [tile parity][weight block r][kb][token]: fl32(s_W[r, kb] * s_X[token, kb])
  alignas(16) float fs[2][2][MAX_KB][NMAX];
  float amax[4][NMAX];            // [lane quadrant][token] (phase 1)
};

constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Smem);
static_assert(SMEM_BYTES <= 227 * 1024, "narrow kernel shared memory");

// rows of a group handled by the narrow tile: see gg::narrow_part
__device__ __forceinline__ int narrow_rows(int rows) { return gg::narrow_part(rows, NMAX); }

struct NTile {
  int g, n, row0, rows;   // row0: first token row in the A-side tensor; rows: 1..64
  bool shared;
};

template <int PHASE>
__device__ __forceinline__ NTile decode_ntile(const Smem& sm, const Args& a, int t, int n_tiles) {
  NTile tl;
  const int G = a.N_r + 1;
  tl.g = gg::find_group(sm.tile_start, G, t);
  tl.n = t - sm.tile_start[tl.g];
  tl.shared = tl.g == a.N_r;
  const int grows = tl.shared ? a.T : sm.off[tl.g + 1] - sm.off[tl.g];
  const int base = tl.shared ? (PHASE == 1 ? 0 : a.P) : sm.off[tl.g];
  tl.rows = narrow_rows(grows);
  tl.row0 = base + (grows - tl.rows);
  (void)n_tiles;
  return tl;
}

// Factor table of a tile: fs[par][r][kb][j] = fl32(s_W[r, kb] * s_X[j, kb]),
// r = 0/1 the two weight tiles of the MMA pair (gate/up in phase 1, the two
// 128-channel halves of W_down in phase 2), j the tile's token. Tokens past
// the tile's rows get 0. Thread `tid` of the 256 epilogue threads fills
// entries tid, tid + 256, ... in token-fastest order.
template <int PHASE>
__device__ __forceinline__ void stage_factors(Smem& sm, const Args& a, const NTile& tl, uint32_t par,
                                              int KB, int tid) {
  const float* xsrc;
  const float* w0;
  const float* w1;
  if (PHASE == 1) {
    const int KBi = a.I / BK;
    xsrc = (tl.shared ? a.xs : a.xs_perm) + static_cast<size_t>(tl.row0) * KB;
    w0 = a.s_gate + static_cast<size_t>(tl.g * KBi + tl.n) * KB;
    w1 = a.s_up + static_cast<size_t>(tl.g * KBi + tl.n) * KB;
  } else {
    const int KBd = a.d / BK;
    xsrc = a.Hs + static_cast<size_t>(tl.row0) * KB;
    w0 = a.s_down + static_cast<size_t>(tl.g * KBd + tl.n * 2) * KB;
    w1 = w0 + KB;
  }
  const int nt = (tl.rows + 15) & ~15;
#pragma unroll 4
  for (int e = tid; e < KB * NMAX; e += EPI_WARPS * 32) {
    const int kb = e / NMAX, j = e % NMAX;
    if (j < nt) {
      const float xv = j < tl.rows ? __ldg(xsrc + static_cast<size_t>(j) * KB + kb) : 0.0f;
      sm.fs[par][0][kb][j] = __ldg(w0 + kb) * xv;
      sm.fs[par][1][kb][j] = __ldg(w1 + kb) * xv;
    }
  }
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// acc[i] += f.{x,y,z,w}[i] * r[i] for four consecutive values
__device__ __forceinline__ void fma4(float* acc, const float4 f, const uint32_t* r) {
  acc[0] = fmaf(f.x, __uint_as_float(r[0]), acc[0]);
  acc[1] = fmaf(f.y, __uint_as_float(r[1]), acc[1]);
  acc[2] = fmaf(f.z, __uint_as_float(r[2]), acc[2]);
  acc[3] = fmaf(f.w, __uint_as_float(r[3]), acc[3]);
}

struct EpiCtx {
  uint32_t tq;       // TMEM address of the warp's lane quadrant, column 0
  int q, half, lane, KB;
  uint32_t par;
  volatile int* abort;
};

// One tile of the epilogue for an MMA width N = 2 * NC. The thread owns one
// weight row (TMEM lane) and 2 * NC accumulators in two ranges of NC columns:
//   phase 1: gate and up of tokens half*NC .. +NC (SwiGLU pairs them);
//   phase 2: tokens 0 .. 2*NC of weight tile `half`.
// Per K block: read the two ranges, release the buffer, then one FMA per
// value with the staged factors (128-bit broadcast loads).
template <int PHASE, int NC>
__device__ __forceinline__ bool epi_tile(Smem& sm, const Args& a, const NTile tl, const EpiCtx x,
                                         int& kbg) {
  constexpr int NV = 2 * NC;
  const int j0 = PHASE == 1 ? x.half * NC : 0;
  const uint32_t colA = PHASE == 1 ? j0 : x.half * 64;
  const uint32_t colB = PHASE == 1 ? 64 + j0 : x.half * 64 + NC;
  // shared-memory addresses of the factor rows of the two ranges at kb = 0
  const uint32_t fA = smem_u32(PHASE == 1 ? &sm.fs[x.par][0][0][j0] : &sm.fs[x.par][x.half][0][0]);
  const uint32_t fB = smem_u32(PHASE == 1 ? &sm.fs[x.par][1][0][j0] : &sm.fs[x.par][x.half][0][NC]);
  float acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.0f;
  for (int kb = 0; kb < x.KB; ++kb, ++kbg) {
    const int buf = kbg % NBUF;
    const uint32_t tph = (kbg / NBUF) & 1;
    if (!warp_wait(&sm.tfull[buf], tph, x.abort)) return false;
    tc_fence_after();
    const uint32_t tb = x.tq + buf * 128;
    const uint32_t pa = fA + kb * (NMAX * 4), pb = fB + kb * (NMAX * 4);
    if (NC < 32) {
      // both ranges in flight at once
      uint32_t r[NV];
#pragma unroll
      for (int p = 0; p < NC / 8; ++p) {
        tmem_ld8_async(tb + colA + 8 * p, &r[8 * p]);
        tmem_ld8_async(tb + colB + 8 * p, &r[NC + 8 * p]);
      }
      tmem_wait_ld(r);
      tc_fence_before();
      __syncwarp();
      if (x.lane == 0) mbar_arrive(&sm.tempty[buf]);
#pragma unroll
      for (int p = 0; p < NC / 4; ++p) {
        fma4(&acc[4 * p], lds_f4(pa + 16 * p), &r[4 * p]);
        fma4(&acc[NC + 4 * p], lds_f4(pb + 16 * p), &r[NC + 4 * p]);
      }
    } else {
      // one range at a time, so that 2 x 64 accumulators and loaded values
      // stay within the register budget
      uint32_t r[NC];
#pragma unroll
      for (int p = 0; p < NC / 8; ++p) tmem_ld8_async(tb + colA + 8 * p, &r[8 * p]);
      tmem_wait_ld(r);
#pragma unroll
      for (int p = 0; p < NC / 4; ++p) fma4(&acc[4 * p], lds_f4(pa + 16 * p), &r[4 * p]);
#pragma unroll
      for (int p = 0; p < NC / 8; ++p) tmem_ld8_async(tb + colB + 8 * p, &r[8 * p]);
      tmem_wait_ld(r);
      tc_fence_before();
      __syncwarp();
      if (x.lane == 0) mbar_arrive(&sm.tempty[buf]);
#pragma unroll
      for (int p = 0; p < NC / 4; ++p) fma4(&acc[NC + 4 * p], lds_f4(pb + 16 * p), &r[4 * p]);
    }
  }

  const int c = x.q * 32 + x.lane;   // weight row within the 128-row tile
  if (PHASE == 1) {
    // SwiGLU for (channel c, token j0 + i), then per token the max-abs over
    // the tile's 128 channels: across the warp's lanes with shuffles, then
    // across the four lane-quadrant warps through shared memory.
    float h[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) h[i] = gg::silu_fast(acc[i]) * acc[NC + i];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      float m = fabsf(h[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (x.lane == 0) sm.amax[x.q][j0 + i] = m;
    }
    __syncwarp();
    if (x.lane == 0) mbar_arrive(&sm.xbar);
    if (!warp_wait(&sm.xbar, x.par, x.abort)) return false;
    const int KBi = a.I / BK;
    const size_t col = static_cast<size_t>(tl.n) * 128 + c;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int tok = j0 + i;
      const float am = fmaxf(fmaxf(sm.amax[0][tok], sm.amax[1][tok]), fmaxf(sm.amax[2][tok], sm.amax[3][tok]));
      const float s = tile_scale(am);
      if (tok < tl.rows) {
        // H rows: routed rows as in xq_perm, then the shared expert's T rows
        const size_t hrow = static_cast<size_t>((tl.shared ? a.P : 0) + tl.row0 + tok);
        // the scale follows the stored rule; the code multiplies by its reciprocal
        a.H[hrow * a.I + col] = static_cast<uint8_t>(e4m3x2(h[i] * __fdiv_rn(1.0f, s), 0.0f) & 0xFF);
        if (c == 0) a.Hs[hrow * KBi + tl.n] = s;
      }
    }
  } else {
    // output channel n*256 + half*128 + c of each token: a warp writes 32
    // consecutive channels (128 bytes) of one token at a time
    const int ch = tl.n * 256 + x.half * 128 + c;
    float* y = (tl.shared ? a.y_shared + static_cast<size_t>(tl.row0 - a.P) * a.d
                          : a.y_perm + static_cast<size_t>(tl.row0) * a.d) + ch;
#pragma unroll
    for (int j = 0; j < NV; ++j)
      if (j < tl.rows) y[static_cast<size_t>(j) * a.d] = acc[j];
  }
  return true;
}

template <int PHASE>
__global__ void __launch_bounds__(THREADS, 1)
    narrow_gemm_kernel(const __grid_constant__ CUtensorMap tm_tok, const __grid_constant__ CUtensorMap tm_toks,
                       const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                       const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(tiles + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int G = a.N_r + 1;
  const int KB = (PHASE == 1 ? a.d : a.I) / BK;
  const int n_tiles = PHASE == 1 ? a.I / 128 : a.d / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], EPI_WARPS);
    }
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.sbar, EPI_WARPS);
    mbar_init(&sm.xbar, EPI_WARPS);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_tok);
    tma_prefetch_desc(&tm_toks);
    tma_prefetch_desc(&tm_w0);
    tma_prefetch_desc(&tm_w1);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i <= a.N_r; i += THREADS) sm.off[i] = a.offsets[i];
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += THREADS) {
    const int rows = g == a.N_r ? a.T : sm.off[g + 1] - sm.off[g];
    sm.tile_start[g] = narrow_rows(rows) > 0 ? n_tiles : 0;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix sum of tile counts, in place
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int i = base + lane;
      const int v = i < G ? sm.tile_start[i] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      if (i < G) sm.tile_start[i] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      sm.tile_start[G] = carry;
      sm.total_tiles = carry;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int total = sm.total_tiles;
  volatile int* abort = &sm.abort;

  if (warp < EPI_WARP0) {
    regs_decrease<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ TMA producer
      int armed[STAGES];
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t pol_w = l2_policy_evict_last();
      for (int t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
        const NTile tl = decode_ntile<PHASE>(sm, a, t, n_tiles);
        const CUtensorMap* xm = (PHASE == 1 && tl.shared) ? &tm_toks : &tm_tok;
        const int w0 = PHASE == 1 ? tl.g * a.I + tl.n * 128 : tl.g * a.d + tl.n * 256;
        const int w1 = PHASE == 1 ? w0 : w0 + 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort)) break;
          uint8_t* dst = tiles + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&sm.full[stage], STAGE_BYTES);
          tma_load_2d_hint(dst, &tm_w0, &sm.full[stage], kb * BK, w0, pol_w);
          tma_load_2d_hint(dst + A_BYTES, &tm_w1, &sm.full[stage], kb * BK, w1, pol_w);
          tma_load_2d(dst + 2 * A_BYTES, xm, &sm.full[stage], kb * BK, tl.row0);
          armed[stage] = phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort) {
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (armed[s] >= 0) mbar_wait(&sm.full[s], armed[s], &never, 100000000ull);
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int kbg = 0;          // K blocks issued so far (selects the partial buffer)
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const NTile tl = decode_ntile<PHASE>(sm, a, t, n_tiles);
        const int nt = (tl.rows + 15) & ~15;
        const uint32_t idesc = make_idesc(0, 0, 128, nt);
        for (int kb = 0; kb < KB; ++kb, ++kbg) {
          const int buf = kbg % NBUF;
          const uint32_t tph = (kbg / NBUF) & 1;
          if (!mbar_wait(&sm.tempty[buf], tph ^ 1, abort)) { ok = false; break; }
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(tiles + stage * STAGE_BYTES);
          const uint64_t bd = sw128_kmajor_desc(base + 2 * A_BYTES);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t ad = sw128_kmajor_desc(base + h * A_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              umma_f8f6f4(tmem + buf * 128 + h * 64, ad + 2 * k, bd + 2 * k, idesc, k > 0);
          }
          umma_commit(&sm.empty[stage]);
          umma_commit(&sm.tfull[buf]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      umma_commit(&sm.drain);
      volatile int never = 0;
      mbar_wait(&sm.drain, 0, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------ epilogue
    regs_increase<REGS_EPI>();
    const int ew = warp - EPI_WARP0;           // 0..7
    const int q = warp & 3;                    // TMEM lane quadrant
    const int half = ew >> 2;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int kbg = 0;
    uint32_t par = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const NTile tl = decode_ntile<PHASE>(sm, a, t, n_tiles);
      stage_factors<PHASE>(sm, a, tl, par, KB, ew * 32 + lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sbar);
      if (!warp_wait(&sm.sbar, par, abort)) break;
      const EpiCtx ctx{tq, q, half, lane, KB, par, abort};
      bool ok = false;
      switch ((tl.rows + 15) >> 4) {   // MMA width N = 16, 32, 48 or 64
        case 1: ok = epi_tile<PHASE, 8>(sm, a, tl, ctx, kbg); break;
        case 2: ok = epi_tile<PHASE, 16>(sm, a, tl, ctx, kbg); break;
        case 3: ok = epi_tile<PHASE, 24>(sm, a, tl, ctx, kbg); break;
        default: ok = epi_tile<PHASE, 32>(sm, a, tl, ctx, kbg); break;
      }
      if (!ok) break;
      par ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace gn
}  // namespace moe
