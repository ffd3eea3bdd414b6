// Grouped FP8 GEMM for all expert FFNs of the layer (routed experts on the
// permuted rows, the shared expert on all tokens).
//
// Numerics ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8 bullet: E4M3
// operands, 1x128 activation tiles, 128x128 weight blocks, FP32 promotion of
// the accumulation every N_c = 128): every product is
//     C[m, n] = sum_kb  s_A[m, kb] * s_W[n/128, kb] * P_kb[m, n],
//     P_kb = A[m, kb*128 : kb*128+128] . W[n, kb*128 : kb*128+128],
// The tensor cores produce each 128-wide partial P_kb into a fresh TMEM
// buffer (four tcgen05.mma kind::f8f6f4 of K = 32). The epilogue warps read it
// with tcgen05.ld, multiply by the two FP32 scales and add it to an FP32
// register accumulator. Only one K block ever sums inside the tensor core. On
// H800 the promotion moved the partial sums into CUDA-core registers; here
// TMEM plays that role with two partial buffers in flight, so the next block's
// MMAs overlap the FMAs of the current one.
//
// Structure (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 0     TMA producer: A tile 128 x 128 and B tile 256 x 128 per K block
//              (128-byte swizzle), 4-stage ring (3 in phase 2); with the
//              gather variant the A rows come straight from the unpermuted
//              activations by tile::gather4 (four rows per load).
//   warps 1, 3 MMA issuers (lane 0 of each): warp 1 issues the even K blocks
//              into TMEM buffer 0, warp 3 the odd ones into buffer 1, so each
//              waits only on its own buffer's release. Warp 1 owns the TMEM
//              allocation (512 columns = 2 x 256).
//   warp 2     idle (it completes the first warpgroup).
//   warps 4-11 epilogue: warp w reads TMEM lanes 32*(w%4).. (rows), and
//              (w-4)/4 selects the column half. Each thread keeps 128 FP32
//              accumulators, so the epilogue warpgroups take 224 registers
//              per thread and the first warpgroup gives its share back (56).
//              Each partial is read 32 columns at a time with two reads in
//              flight, and the buffer is released as soon as the last two
//              reads have landed in registers, before their FMAs.
//
// What paces the K loop: four MMAs of N = 256 take about 513 cycles, but a
// buffer goes round MMA completion -> read-back of 128 x 256 FP32 values ->
// FMAs -> release in more than that, and with only two buffers (TMEM holds
// 512 columns) the round trip is not hidden: a K block takes about 1.2K
// cycles at d = 7168.
//
// Two launches:
//   phase 1: per tile (group g, 128 rows, 128 intermediate channels n):
//            B = [W_gate rows n*128..+128 ; W_up rows n*128..+128], N = 256.
//            Epilogue: SwiGLU a = silu(G) * U, 1x128 requantisation to E4M3
//            (the tile is exactly one 128-channel scale tile), written to H.
//   phase 2: per tile (group g, 128 rows, 256 output channels):
//            A = H, B = W_down rows; the FP32 accumulators are rounded to
//            bf16 and leave through shared memory and TMA stores (the
//            combine adds them to the residual in FP32). The backward's
//            GEMMs run this phase on its own with FP32 outputs, and in a
//            K-grouped mode where every group has its own K range.
// Tiles are numbered group-major (shared expert last), then row tile, then
// column tile. The first wave is dealt by block index; after it each CTA
// claims the next number from a counter in the workspace, so the tiles in
// flight stay a window of about one wave and those sharing weight tiles and
// activation rows read them from L2 at the same time.
//
// Narrow tiles: a group of only 1..64 rows (decode batches: a few tokens per
// expert) would pay a 128 x 256 partial read-back per K block for them. Its
// tile swaps the MMA's roles instead: the two 128-row weight tiles of the
// stage are M, the group's N = rows rounded up to 16 token rows are N (two
// N <= 64 MMAs into columns 0 and 128 of the partial buffer), and the
// epilogue owns one weight row per thread with a per-token scale table in
// shared memory: half the TMEM read-back, and less power for the same
// weight stream. Its TMA loads are the wide tile's.
//
// The per-tile epilogue tail sits between two tiles' K loops, and the MMAs can
// only run two K blocks ahead of it, so it is kept short: SwiGLU and the
// requantisation use the fast exponential/division (branch-free, a few
// instructions each, so the unrolled tail stays small), and the phase-2
// output is handed to TMA instead of 32 scattered stores per thread.
#include <algorithm>

#include "host.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 384;
constexpr int EPI_THREADS = 256;
constexpr int EPI_WARPS = 8;
constexpr int EPI_WARP0 = 4;     // first epilogue warp
// launch at 168 registers (65536 / 384, rounded down to 8); then
// 128 * 56 + 256 * 224 = 384 * 168, and 56 + 2 * 224 <= 512 per sub-partition
constexpr uint32_t REGS_CTRL = 56;
constexpr uint32_t REGS_EPI = 224;
constexpr int MAX_GROUPS = 1025;
constexpr int TILE_RING = 4;     // tile numbers the producer may publish ahead of the consumers
constexpr int MMA_THREADS = 2;   // MMA issuers (lane 0 of warps 1 and 3): even and odd K blocks
constexpr uint32_t TMEM_COLS = 512;
// narrow tiles: at most 64 token rows; K blocks of the tile's token-scale
// table (phase 1: d/128, phase 2: I/128; phase 2 has less room beside the
// output staging)
constexpr int NMAX = 64;
constexpr int MAX_KB_N1 = 56;
constexpr int MAX_KB_N2 = 24;
// phase-2 output staging: per epilogue warp two 32 x 32 FP32 boxes
constexpr int Y_BOX = 32;
constexpr int Y_BOX_BYTES = Y_BOX * Y_BOX * 4;
constexpr int Y_STAGING_BYTES = EPI_WARPS * 2 * Y_BOX_BYTES;

template <int PHASE>
struct Cfg {
  static constexpr int STAGES = PHASE == 1 ? 4 : 3;
  static constexpr int STAGING = PHASE == 1 ? 0 : Y_STAGING_BYTES;
  static constexpr int TAB_KB = PHASE == 1 ? MAX_KB_N1 : MAX_KB_N2;
};

struct Args {
  const int32_t* offsets;
  int N_r, T, P, d, I;
  int narrow_max;            // groups of 1..narrow_max rows run as narrow tiles (0: none)
  const float* xs_perm;
  const float* xs;
  const float* s_gate;
  const float* s_up;
  const float* s_down;
  uint8_t* H;
  float* Hs;
  void* y_perm;              // phase-2 output rows: FP32, or bf16 when y_bf16
  void* y_shared;
  int y_bf16;
  int* tile_counter;         // zeroed before the launch; tiles past the first wave are claimed from it
  const int32_t* sorted_token;  // non-null: routed rows are read from xq/xs at these tokens (no xq_perm)
  // K-grouped (phase 2 only): N_r + 1 groups share A's T rows and B's rows;
  // group g contracts over K elements offsets[g]..offsets[g+1] (multiples of
  // 128; I = the total K) and writes output rows g*T..g*T+T
  int kgrouped;
};

template <int STAGES, int TAB_KB>
struct Smem {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain[2];
  uint64_t xbar;      // epilogue exchange of max-abs partials (phase 1)
  uint64_t sbar;      // narrow tile: token-scale table staged (8 warps)
  uint64_t dbar;      // narrow tile: token-scale table no longer read (8 warps)
  uint64_t rfull[TILE_RING];   // tile number published by the producer
  uint64_t rfree[TILE_RING];   // read by the 2 MMA threads and the 8 epilogue warps
  int ring[TILE_RING];         // tile numbers in claim order; -1 ends the CTA's work
  uint32_t tmem_base;
  int abort;
  int total_tiles;
  int off[MAX_GROUPS + 1];
  int tile_start[MAX_GROUPS + 1];
  // wide tiles: [tile parity][column half][row]; narrow tiles use each
  // parity's 256 floats as [lane quadrant][token]
  float amax_x[2][2][BM];
  alignas(16) float xs_tab[TAB_KB][NMAX];  // narrow tile: [kb][token] activation scales
};

template <int PHASE>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<PHASE>::STAGES * STAGE_BYTES + Cfg<PHASE>::STAGING +
         sizeof(Smem<Cfg<PHASE>::STAGES, Cfg<PHASE>::TAB_KB>);
}
static_assert(smem_bytes<1>() <= 227 * 1024 && smem_bytes<2>() <= 227 * 1024, "shared memory per CTA");

// Rows of a group that form a narrow tile: the whole group when it has
// 1..narrow_max rows. (Measured: a narrow tile for the remainder of a larger
// group is no cheaper than the padded 128-row tile, since an MMA with N <= 64
// costs nearly as much as one with N = 256.)
__device__ __forceinline__ int narrow_part(int rows, int narrow_max) {
  return rows <= narrow_max ? rows : 0;
}

__device__ __forceinline__ int find_group(const int* start, int G, int t) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Tile {
  int g, m, n, rows, row0;  // rows of the group; row0 = first row of the group in its A tensor
  int orow0;                // first output row of the group (row0 unless K-grouped)
  int k0, kb;               // the tile's K blocks: k0 .. k0 + kb
  int mrows;                // narrow tile: its rows (1..narrow_max, the whole group)
  bool shared, narrow;
};

template <int PHASE, typename S>
__device__ __forceinline__ Tile decode_tile(const S& sm, const Args& a, int t, int n_tiles) {
  Tile tl;
  const int G = a.N_r + 1;
  tl.g = find_group(sm.tile_start, G, t);
  const int local = t - sm.tile_start[tl.g];
  tl.m = local / n_tiles;
  tl.n = local - tl.m * n_tiles;
  tl.k0 = 0;
  tl.kb = (PHASE == 1 ? a.d : a.I) / BK;
  if (PHASE == 2 && a.kgrouped) {
    tl.shared = false;
    tl.rows = a.T;
    tl.row0 = 0;
    tl.orow0 = tl.g * a.T;
    const int lo = sm.off[tl.g], hi = sm.off[tl.g + 1];
    if (lo < 0 || hi < lo || hi > a.I || lo % BK != 0 || hi % BK != 0) {
      set_device_error(MOE_ERR_INVALID_ARG);   // every role decodes the same: no K blocks
      tl.kb = 0;
    } else {
      tl.k0 = lo / BK;
      tl.kb = (hi - lo) / BK;
    }
    tl.mrows = 0;
    tl.narrow = false;
    return tl;
  }
  tl.shared = tl.g == a.N_r;
  if (tl.shared) {
    tl.rows = a.T;
    tl.row0 = PHASE == 1 ? 0 : a.P;  // phase 2 reads H, where shared rows follow the routed ones
  } else {
    tl.row0 = sm.off[tl.g];
    tl.rows = sm.off[tl.g + 1] - tl.row0;
  }
  tl.orow0 = tl.row0;
  tl.mrows = narrow_part(tl.rows, a.narrow_max);  // a narrow group has one row tile
  tl.narrow = tl.mrows > 0;
  return tl;
}

// silu(x) = x / (1 + e^-x) with the fast exponential and division: branch-free
// (x -> -inf gives e^-x = inf and x / inf = -0, the limit).
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// Two floats rounded to bf16 (round to nearest even), packed low | high << 16.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  return static_cast<uint32_t>(float_to_bf16_bits(lo)) | (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
}

// 2-D tiled store of one box from shared memory (bulk async group).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(m),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
// Four rows y0..y3 of a 2-D tensor (box: one row of 128 bytes) into four
// consecutive 128-byte rows of shared memory, completion counted on `bar`.
// The tensor map's 128-byte swizzle is applied by shared-memory address, so
// four such loads at 512-byte steps from a 1024-byte aligned base lay out 16
// rows exactly as one 16-row tile load would.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y0, int y1,
                                            int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N bulk groups of this thread still read shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// acc[i] += fl32(t_i * w) * r[i] for four consecutive values (t: staged
// activation scales, w: the weight block's scale; the factor is rounded to
// FP32 before the FMA, as in the wide tiles)
__device__ __forceinline__ void fma4(float* acc, const float4 t, float w, const uint32_t* r) {
  acc[0] = fmaf(t.x * w, __uint_as_float(r[0]), acc[0]);
  acc[1] = fmaf(t.y * w, __uint_as_float(r[1]), acc[1]);
  acc[2] = fmaf(t.z * w, __uint_as_float(r[2]), acc[2]);
  acc[3] = fmaf(t.w * w, __uint_as_float(r[3]), acc[3]);
}

struct NarrowCtx {
  uint32_t tq;                  // TMEM address of the warp's lane quadrant, column 0
  int q, half, lane, tid, KB;   // tid: 0..255 over the epilogue warps
  volatile int* abort;
};

// Epilogue of a narrow tile: a group of 1..64 rows, computed with the
// weights as the MMA's M side, so TMEM lane = weight row (channel) and TMEM
// column = token. N = 2 * NC token columns (the rows rounded up to 16).
//   phase 1: columns [0, N) hold W_gate x X^T and [128, 128 + N) W_up x X^T of
//            the tile's 128 channels; the thread (channel c) owns tokens
//            half*NC .. +NC of both, pairs them in SwiGLU and requantises each
//            token's 128 channels (max-abs across lanes, then across the four
//            lane-quadrant warps).
//   phase 2: columns [half*128, half*128 + N) hold W_down rows n*256 +
//            half*128 .. +128 x H^T; the thread owns all N tokens of one
//            output channel.
// The activation scales of the tile are staged once per tile as a [kb][token]
// table, so each value costs one FP32 multiply and one FMA.
template <int PHASE, int NC, typename S>
__device__ __forceinline__ bool narrow_tile(S& sm, const Args& a, const Tile tl, const NarrowCtx x, int& buf,
                                            uint32_t& tphase, uint32_t& xpar, int& nn) {
  constexpr int NV = 2 * NC;
  const int KBd = a.d / BK, KBi = a.I / BK;
  const int r0 = tl.row0 + tl.m * BM;   // first row of the tile in the A tensor

  // stage the table once the previous narrow tile's table is read by all warps
  if (nn > 0 && !warp_wait(&sm.dbar, (nn - 1) & 1, x.abort)) return false;
  {
    const bool gathered = PHASE == 1 && !tl.shared && a.sorted_token != nullptr;
    const float* xsrc = PHASE == 1 ? (tl.shared ? a.xs : a.xs_perm) + static_cast<size_t>(r0) * KBd
                                   : a.Hs + static_cast<size_t>(r0) * KBi;
    for (int e = x.tid; e < x.KB * NMAX; e += EPI_THREADS) {
      const int kb = e / NMAX, j = e % NMAX;
      float v = 0.0f;
      if (j < tl.mrows)
        v = gathered ? __ldg(a.xs + static_cast<size_t>(__ldg(a.sorted_token + r0 + j)) * KBd + kb)
                     : __ldg(xsrc + static_cast<size_t>(j) * x.KB + kb);
      sm.xs_tab[kb][j] = v;
    }
  }
  __syncwarp();
  if (x.lane == 0) mbar_arrive(&sm.sbar);
  if (!warp_wait(&sm.sbar, nn & 1, x.abort)) return false;
  ++nn;

  const int j0 = PHASE == 1 ? x.half * NC : 0;
  const uint32_t colA = PHASE == 1 ? j0 : x.half * 128;
  const uint32_t colB = PHASE == 1 ? 128 + j0 : x.half * 128 + NC;
  const uint32_t tabA = smem_u32(&sm.xs_tab[0][j0]);
  const uint32_t tabB = smem_u32(&sm.xs_tab[0][PHASE == 1 ? j0 : NC]);
  const float* swA;
  const float* swB;
  if (PHASE == 1) {
    swA = a.s_gate + static_cast<size_t>(tl.g * KBi + tl.n) * KBd;
    swB = a.s_up + static_cast<size_t>(tl.g * KBi + tl.n) * KBd;
  } else {
    swA = a.s_down + static_cast<size_t>(tl.g * KBd + tl.n * 2 + x.half) * KBi;
    swB = swA;
  }
  float acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = 0.0f;
  for (int kb = 0; kb < x.KB; ++kb) {
    const float wA = __ldg(swA + kb), wB = __ldg(swB + kb);
    if (!warp_wait(&sm.tfull[buf], tphase, x.abort)) return false;
    tc_fence_after();
    const uint32_t tb = x.tq + buf * BN;
    const uint32_t ta = tabA + kb * (NMAX * 4), tt = tabB + kb * (NMAX * 4);
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
        const float4 t4 = lds_f4(ta + 16 * p);
        fma4(&acc[4 * p], t4, wA, &r[4 * p]);
        fma4(&acc[NC + 4 * p], PHASE == 1 ? t4 : lds_f4(tt + 16 * p), wB, &r[NC + 4 * p]);
      }
    } else {
      // one range at a time, so that 64 accumulators and the loaded values
      // stay within the register budget
      uint32_t r[NC];
#pragma unroll
      for (int p = 0; p < NC / 8; ++p) tmem_ld8_async(tb + colA + 8 * p, &r[8 * p]);
      tmem_wait_ld(r);
#pragma unroll
      for (int p = 0; p < NC / 4; ++p) fma4(&acc[4 * p], lds_f4(ta + 16 * p), wA, &r[4 * p]);
#pragma unroll
      for (int p = 0; p < NC / 8; ++p) tmem_ld8_async(tb + colB + 8 * p, &r[8 * p]);
      tmem_wait_ld(r);
      tc_fence_before();
      __syncwarp();
      if (x.lane == 0) mbar_arrive(&sm.tempty[buf]);
#pragma unroll
      for (int p = 0; p < NC / 4; ++p) fma4(&acc[NC + 4 * p], lds_f4(tt + 16 * p), wB, &r[4 * p]);
    }
    buf ^= 1;
    if (buf == 0) tphase ^= 1;
  }
  __syncwarp();
  if (x.lane == 0) mbar_arrive(&sm.dbar);   // this warp no longer reads the table

  const int c = x.q * 32 + x.lane;           // weight row within the 128-row tile
  if (PHASE == 1) {
    float hv[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) hv[i] = silu_fast(acc[i]) * acc[NC + i];
    float* am = &sm.amax_x[xpar][0][0];      // [lane quadrant][token]
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      float m = fabsf(hv[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (x.lane == 0) am[x.q * NMAX + j0 + i] = m;
    }
    __syncwarp();
    if (x.lane == 0) mbar_arrive(&sm.xbar);
    if (!warp_wait(&sm.xbar, xpar, x.abort)) return false;
    xpar ^= 1;
    const size_t col = static_cast<size_t>(tl.n) * 128 + c;
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const int tok = j0 + i;
      const float m = fmaxf(fmaxf(am[tok], am[NMAX + tok]), fmaxf(am[2 * NMAX + tok], am[3 * NMAX + tok]));
      const float sc = tile_scale(m);
      if (tok < tl.mrows) {
        // H rows: routed rows as in xq_perm, then the shared expert's T rows
        const size_t hrow = static_cast<size_t>((tl.shared ? a.P : 0) + r0 + tok);
        // the scale follows the stored rule; the code multiplies by its reciprocal
        a.H[hrow * a.I + col] = static_cast<uint8_t>(e4m3x2(hv[i] * __fdiv_rn(1.0f, sc), 0.0f) & 0xFF);
        if (c == 0) a.Hs[hrow * KBi + tl.n] = sc;
      }
    }
  } else {
    // output channel n*256 + half*128 + c of each token: a warp writes 32
    // consecutive channels of one token at a time
    const size_t at = (tl.shared ? static_cast<size_t>(r0 - a.P) : static_cast<size_t>(r0)) * a.d +
                      (tl.n * BN + x.half * 128 + c);
    void* ybase = tl.shared ? a.y_shared : a.y_perm;
    if (a.y_bf16) {
      uint16_t* y = static_cast<uint16_t*>(ybase) + at;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (j < tl.mrows) y[static_cast<size_t>(j) * a.d] = float_to_bf16_bits(acc[j]);
    } else {
      float* y = static_cast<float*>(ybase) + at;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (j < tl.mrows) y[static_cast<size_t>(j) * a.d] = acc[j];
    }
  }
  return true;
}

template <int PHASE>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                        const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_ys,
                        const __grid_constant__ CUtensorMap tm_xg, const Args a) {
  constexpr int STAGES = Cfg<PHASE>::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = tiles + STAGES * STAGE_BYTES;   // 1024-aligned (phase 2 only)
  using SmemT = Smem<STAGES, Cfg<PHASE>::TAB_KB>;
  SmemT& sm = *reinterpret_cast<SmemT*>(staging + Cfg<PHASE>::STAGING);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int G = a.N_r + 1;
  const int KB = (PHASE == 1 ? a.d : a.I) / BK;            // K blocks per tile
  const int n_tiles = PHASE == 1 ? a.I / 128 : a.d / BN;    // column tiles per row tile

  // ---- setup: barriers, TMEM, the tile table
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], EPI_WARPS);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    mbar_init(&sm.xbar, EPI_WARPS);
    mbar_init(&sm.sbar, EPI_WARPS);
    mbar_init(&sm.dbar, EPI_WARPS);
    for (int i = 0; i < TILE_RING; ++i) {
      mbar_init(&sm.rfull[i], 1);
      mbar_init(&sm.rfree[i], MMA_THREADS + EPI_WARPS);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_b0);
    tma_prefetch_desc(&tm_b1);
    if (PHASE == 1 && a.sorted_token != nullptr) tma_prefetch_desc(&tm_xg);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  const bool kg = PHASE == 2 && a.kgrouped;
  for (int i = threadIdx.x; i <= (kg ? G : a.N_r); i += THREADS) sm.off[i] = a.offsets[i];
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += THREADS) {
    const int rows = (kg || g == a.N_r) ? a.T : sm.off[g + 1] - sm.off[g];
    sm.tile_start[g] = ((rows + BM - 1) / BM) * n_tiles;
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
    if (warp == 0) {
      // ------------------------------------------------ TMA producer
      // Lane 0 owns the barriers and the schedule. When the routed rows are
      // gathered from xq (sorted_token given), every lane also issues one
      // four-row gather per K block: lane i fetches rows 4i..4i+3 of the A tile.
      int armed[STAGES];
      for (int s = 0; s < STAGES; ++s) armed[s] = -1;
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t pol_w = l2_policy_evict_last();
      // Dynamic schedule: the first wave takes tiles blockIdx.x, later tiles
      // are claimed from a global counter when this CTA's previous tile has
      // all its loads issued, so the CTAs stay within about one wave of each
      // other and tiles that share weight blocks and activation rows run at
      // the same time (their operands meet in L2). Each claimed number is
      // published to the MMA threads and the epilogue through a ring in
      // shared memory; -1 ends the CTA's work.
      int rslot = 0;
      uint32_t rph = 0;
      int t = blockIdx.x;
      for (;;) {
        int tt = -1, okr = 1;
        if (lane == 0) {
          okr = mbar_wait(&sm.rfree[rslot], rph ^ 1, abort) ? 1 : 0;
          if (okr) {
            tt = t < total ? t : -1;
            sm.ring[rslot] = tt;
            mbar_arrive(&sm.rfull[rslot]);
            if (++rslot == TILE_RING) {
              rslot = 0;
              rph ^= 1;
            }
          }
        }
        okr = __shfl_sync(0xffffffffu, okr, 0);
        tt = __shfl_sync(0xffffffffu, tt, 0);
        if (!okr || tt < 0 || *abort) break;
        const Tile tl = decode_tile<PHASE>(sm, a, tt, n_tiles);
        const bool gather = PHASE == 1 && !tl.shared && a.sorted_token != nullptr;
        const CUtensorMap* am = (PHASE == 1 && tl.shared) ? &tm_x : &tm_a;
        const int arow = tl.row0 + tl.m * BM;
        int tok[4] = {0, 0, 0, 0};
        // gathered tiles fetch only the four-row groups holding rows of the
        // group (the tile's other rows keep stale data; their products are
        // never stored)
        const int live = gather ? min(BM, tl.rows - tl.m * BM) : 0;
        const int n_g4 = (live + 3) / 4;
        if (gather && lane < n_g4) {
          const int last = tl.row0 + tl.rows - 1;
#pragma unroll
          for (int i = 0; i < 4; ++i) tok[i] = __ldg(a.sorted_token + min(arow + 4 * lane + i, last));
        }
        const uint32_t stage_bytes = gather ? STAGE_BYTES - A_BYTES + n_g4 * 4 * BK : STAGE_BYTES;
        for (int kb = 0; kb < tl.kb; ++kb) {
          const int kx = (tl.k0 + kb) * BK;
          int okw = 1;
          uint8_t* dst = tiles + stage * STAGE_BYTES;
          if (lane == 0) {
            okw = mbar_wait(&sm.empty[stage], phase ^ 1, abort) ? 1 : 0;
            if (okw) {
              mbar_arrive_expect_tx(&sm.full[stage], stage_bytes);
              if (!gather) tma_load_2d(dst, am, &sm.full[stage], kx, arow);
              if (PHASE == 1) {
                const int wrow = tl.g * a.I + tl.n * 128;
                tma_load_2d_hint(dst + A_BYTES, &tm_b0, &sm.full[stage], kx, wrow, pol_w);
                tma_load_2d_hint(dst + A_BYTES + B_BYTES / 2, &tm_b1, &sm.full[stage], kx, wrow, pol_w);
              } else {
                const int wrow = (kg ? 0 : tl.g * a.d) + tl.n * BN;
                tma_load_2d_hint(dst + A_BYTES, &tm_b0, &sm.full[stage], kx, wrow, pol_w);
              }
              armed[stage] = phase;
            }
          }
          okw = __shfl_sync(0xffffffffu, okw, 0);   // also orders the copies after the expected bytes
          if (!okw) break;
          if (gather && lane < n_g4)
            tma_gather4(dst + lane * 4 * BK, &tm_xg, &sm.full[stage], kx, tok[0], tok[1], tok[2], tok[3]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (lane == 0) t = static_cast<int>(gridDim.x) + atomicAdd(a.tile_counter, 1);
      }
      if (lane == 0 && *abort) {
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (armed[s] >= 0) mbar_wait(&sm.full[s], armed[s], &never, 100000000ull);
      }
      __syncwarp();
    } else if ((warp == 1 || warp == 3) && lane == 0) {
      // ------------------------------------------------ MMA issuers
      // Issuing a K block's four MMAs and two commits, after two barrier
      // checks, is a chain of long-latency instructions for one thread
      // (about a microsecond's worth of issue latency next to the epilogue's
      // FMA streams, measured). Two threads on different SM sub-partitions
      // take alternate K blocks of the CTA's sequence: thread j the blocks
      // k = j (mod 2), which use TMEM buffer j and every other pipeline stage,
      // so their chains overlap while each buffer is still filled and drained
      // in order.
      const int j = warp == 1 ? 0 : 1;
      const uint32_t idesc = make_idesc(0, 0, BM, BN);
      int stage = j;              // stage of this thread's next K block
      uint32_t phase = 0;
      const int buf = j;
      uint32_t tphase = 0;
      uint32_t kpar = 0;          // parity of the CTA's K-block sequence
      bool ok = true;
      int rslot = 0;
      uint32_t rph = 0;
      while (ok) {
        if (!mbar_wait(&sm.rfull[rslot], rph, abort)) break;
        const int t = *reinterpret_cast<volatile int*>(&sm.ring[rslot]);
        mbar_arrive(&sm.rfree[rslot]);
        if (++rslot == TILE_RING) {
          rslot = 0;
          rph ^= 1;
        }
        if (t < 0) break;
        const Tile tl = decode_tile<PHASE>(sm, a, t, n_tiles);
        // narrow tile: the weights are M (two 128-row MMAs into columns 0 and
        // 128 of the buffer), the tile's first N = rows rounded up to 16 token
        // rows of the A stage are N
        const uint32_t idesc_n = make_idesc(0, 0, 128, (tl.mrows + 15) & ~15);
        for (int kb = 0; kb < tl.kb; ++kb, kpar ^= 1) {
          if (kpar != static_cast<uint32_t>(j)) continue;
          // the operands usually land well before the partial buffer is free:
          // check them first, so that only the buffer's wait sits between the
          // epilogue's release and the next MMAs
          // descriptors first: only the waits sit between the epilogue's
          // release and the MMAs
          const uint32_t a_addr = smem_u32(tiles + stage * STAGE_BYTES);
          const uint64_t ad = sw128_kmajor_desc(a_addr);
          const uint64_t bd = sw128_kmajor_desc(a_addr + A_BYTES);
          const uint32_t d_tmem = tmem + buf * BN;
          if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
          if (!mbar_wait(&sm.tempty[buf], tphase ^ 1, abort)) { ok = false; break; }
          tc_fence_after();
          if (!tl.narrow) {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) umma_f8f6f4(d_tmem, ad + 2 * k, bd + 2 * k, idesc, k > 0);
          } else {
            // the two accumulators' K steps interleaved (independent chains
            // overlap in the tensor pipe)
            const uint64_t wd0 = sw128_kmajor_desc(a_addr + A_BYTES);
            const uint64_t wd1 = sw128_kmajor_desc(a_addr + A_BYTES + B_BYTES / 2);
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
              umma_f8f6f4(d_tmem, wd0 + 2 * k, ad + 2 * k, idesc_n, k > 0);
              umma_f8f6f4(d_tmem + 128, wd1 + 2 * k, ad + 2 * k, idesc_n, k > 0);
            }
          }
          umma_commit(&sm.empty[stage]);
          umma_commit(&sm.tfull[buf]);
          stage += 2;                 // this thread's next block is two ahead
          if (stage >= STAGES) {
            stage -= STAGES;
            phase ^= 1;
          }
          tphase ^= 1;
        }
      }
      umma_commit(&sm.drain[j]);
      volatile int never = 0;
      mbar_wait(&sm.drain[j], 0, &never, 100000000ull);
    }
  } else {
    // ------------------------------------------------ epilogue
    regs_increase<REGS_EPI>();
    const int ew = warp - EPI_WARP0;
    const int q = warp & 3;
    const int half = ew >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int buf = 0;
    uint32_t tphase = 0;
    uint32_t xpar = 0;
    int n_narrow = 0;     // narrow tiles done (parity of sbar / dbar)
    const int KBd = a.d / BK, KBi = a.I / BK;
    int rslot = 0;
    uint32_t rph = 0;
    for (;;) {
      if (!warp_wait(&sm.rfull[rslot], rph, abort)) break;
      const int t = *reinterpret_cast<volatile int*>(&sm.ring[rslot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rfree[rslot]);
      if (++rslot == TILE_RING) {
        rslot = 0;
        rph ^= 1;
      }
      if (t < 0) break;
      const Tile tl = decode_tile<PHASE>(sm, a, t, n_tiles);
      if (tl.narrow) {
        NarrowCtx c{tmem + lane_base, q, half, lane, ew * 32 + lane, KB, abort};
        bool ok = false;
        switch ((tl.mrows + 15) >> 4) {   // N = 16, 32, 48 or 64
          case 1: ok = narrow_tile<PHASE, 8>(sm, a, tl, c, buf, tphase, xpar, n_narrow); break;
          case 2: ok = narrow_tile<PHASE, 16>(sm, a, tl, c, buf, tphase, xpar, n_narrow); break;
          case 3: ok = narrow_tile<PHASE, 24>(sm, a, tl, c, buf, tphase, xpar, n_narrow); break;
          default: ok = narrow_tile<PHASE, 32>(sm, a, tl, c, buf, tphase, xpar, n_narrow); break;
        }
        if (!ok) break;
        continue;
      }
      const int rr = tl.m * BM + r;          // row within the group
      const bool valid = rr < tl.rows;
      const int grow = tl.row0 + rr;         // row in the A tensor (and its scales)
      const float* sa_ptr;
      const float* sb0;
      const float* sb1;
      if (PHASE == 1) {
        if (tl.shared || a.sorted_token == nullptr)
          sa_ptr = (tl.shared ? a.xs : a.xs_perm) + static_cast<size_t>(grow) * KBd;
        else   // gathered rows: the scales of the row's token
          sa_ptr = a.xs + static_cast<size_t>(valid ? __ldg(a.sorted_token + grow) : 0) * KBd;
        sb0 = a.s_gate + static_cast<size_t>(tl.g * KBi + tl.n) * KBd;
        sb1 = a.s_up + static_cast<size_t>(tl.g * KBi + tl.n) * KBd;
      } else {   // K-grouped: one B for all groups, the tile's K range from k0
        sa_ptr = a.Hs + static_cast<size_t>(grow) * KBi + tl.k0;
        sb0 = a.s_down + static_cast<size_t>((kg ? 0 : tl.g * KBd) + tl.n * 2 + half) * KBi + tl.k0;
        sb1 = sb0;
      }
      const int KBt = tl.kb;
      float acc[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
      // The row's activation scale (a different cache line for every
      // thread) is loaded two K blocks ahead, the weight block's scales (one
      // line for the whole CTA) one block ahead.
      float sa_n = (valid && KBt > 0) ? __ldg(sa_ptr) : 0.0f;
      float sa_n2 = (valid && KBt > 1) ? __ldg(sa_ptr + 1) : 0.0f;
      float s0_n = KBt > 0 ? __ldg(sb0) : 0.0f, s1_n = KBt > 0 ? __ldg(sb1) : 0.0f;
      bool ok = true;
      for (int kb = 0; kb < KBt; ++kb) {
        const float sa = sa_n, s0 = s0_n, s1 = s1_n;
        sa_n = sa_n2;
        if (kb + 2 < KBt) sa_n2 = valid ? __ldg(sa_ptr + kb + 2) : 0.0f;
        if (kb + 1 < KBt) {
          s0_n = __ldg(sb0 + kb + 1);
          s1_n = __ldg(sb1 + kb + 1);
        }
        if (!warp_wait(&sm.tfull[buf], tphase, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ta = tmem + lane_base + buf * BN;
        // four 32-column chunks of this thread's lane, read two at a time: the
        // first two land together; the third and fourth are issued as soon as
        // the registers of the first and second are consumed, and the buffer
        // is released when they have landed (two read latencies and two chunks
        // of FMAs after the buffer became full).
        //   phase 1: gate columns half*64 + {0, 32}, then up columns 128 + half*64 + {0, 32}
        //   phase 2: columns half*128 + {0, 32, 64, 96}
        const uint32_t c0 = PHASE == 1 ? half * 64 : half * 128;
        const uint32_t c2 = PHASE == 1 ? 128 + half * 64 : half * 128 + 64;
        const float f01 = sa * s0, f23 = sa * s1;   // phase 2: s1 == s0
        uint32_t ra[32], rb[32];
        tmem_ld32_async(ta + c0, ra);
        tmem_ld32_async(ta + c0 + 32, rb);
        tmem_wait_ld2(ra, rb);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fmaf(f01, __uint_as_float(ra[j]), acc[j]);
        tmem_ld32_async(ta + c2, ra);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[32 + j] = fmaf(f01, __uint_as_float(rb[j]), acc[32 + j]);
        tmem_ld32_async(ta + c2 + 32, rb);
        tmem_wait_ld2(ra, rb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[buf]);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[64 + j] = fmaf(f23, __uint_as_float(ra[j]), acc[64 + j]);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[96 + j] = fmaf(f23, __uint_as_float(rb[j]), acc[96 + j]);
        buf ^= 1;
        if (buf == 0) tphase ^= 1;
      }
      if (!ok) break;

      if (PHASE == 1) {
        // SwiGLU on this thread's 64 channels, then the 1x128 requantisation
        // whose max-abs spans both column halves (the partner warp).
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float x = silu_fast(acc[j]) * acc[64 + j];
          acc[j] = x;
          amax = fmaxf(amax, fabsf(x));
        }
        // exchange through shared memory, double-buffered by tile parity; the
        // mbarrier wait is bounded like every other wait here
        sm.amax_x[xpar][half][r] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.xbar);
        if (!warp_wait(&sm.xbar, xpar, abort)) break;
        amax = fmaxf(amax, sm.amax_x[xpar][half ^ 1][r]);
        xpar ^= 1;
        // the scale follows the stored rule; the codes use one reciprocal of
        // it (an E4M3 code can differ from dividing only when x/scale is
        // within an FP32 ulp of a rounding midpoint)
        const float s = tile_scale(amax);
        const float inv = __fdiv_rn(1.0f, s);
        if (valid) {
          const size_t hrow = static_cast<size_t>(tl.shared ? a.P + rr : tl.row0 + rr);
          uint4* dst = reinterpret_cast<uint4*>(a.H + hrow * a.I + tl.n * 128 + half * 64);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int j = i * 16 + k * 4;
              w[k] = e4m3x2(acc[j] * inv, acc[j + 1] * inv) | (e4m3x2(acc[j + 2] * inv, acc[j + 3] * inv) << 16);
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (half == 0) a.Hs[hrow * KBi + tl.n] = s;
        }
      } else {
        // This warp's 32 rows x 128 columns. Rows wholly inside the group go
        // out as four 32 x 32 FP32 boxes: each lane writes its row into a
        // 128-byte-swizzled shared-memory box (16-byte chunk c of row r at
        // chunk c ^ (r % 8): bank-conflict free), and lane 0 hands the box to
        // a TMA store. Two boxes per warp alternate; a box is rewritten only
        // after the store issued two boxes earlier has read it.
        const int row_first = tl.m * BM + q * 32;             // within the group
        const int nvalid = min(Y_BOX, tl.rows - row_first);
        const int col0 = tl.n * BN + half * 128;
        const size_t yrow_at = tl.shared ? static_cast<size_t>(rr) : static_cast<size_t>(tl.orow0 + rr);
        if (a.y_bf16 && nvalid == Y_BOX) {
          // bf16 rows (the layer's expert outputs): two 32 x 64 boxes per
          // warp, each lane's 64 values of a box rounded to bf16 and packed
          // into the row's eight 16-byte chunks (swizzled as the FP32 boxes)
          const CUtensorMap* ym = tl.shared ? &tm_ys : &tm_y;
          const int ytop = tl.shared ? row_first : tl.orow0 + row_first;
          uint8_t* wstage = staging + ew * 2 * Y_BOX_BYTES;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint8_t* box = wstage + c * Y_BOX_BYTES;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float* v = &acc[c * 64 + 8 * i];
              *reinterpret_cast<uint4*>(box + lane * 128 + ((i ^ (lane & 7)) * 16)) =
                  make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]), bf16x2_bits(v[4], v[5]),
                             bf16x2_bits(v[6], v[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(ym, box, col0 + c * 64, ytop);
              bulk_commit();
            }
          }
        } else if (a.y_bf16) {
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(
                static_cast<uint16_t*>(tl.shared ? a.y_shared : a.y_perm) + yrow_at * a.d + col0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float* v = &acc[8 * i];
              dst[i] = make_uint4(bf16x2_bits(v[0], v[1]), bf16x2_bits(v[2], v[3]), bf16x2_bits(v[4], v[5]),
                                  bf16x2_bits(v[6], v[7]));
            }
          }
        } else if (nvalid == Y_BOX) {
          const CUtensorMap* ym = tl.shared ? &tm_ys : &tm_y;
          const int ytop = tl.shared ? row_first : tl.orow0 + row_first;
          uint8_t* wstage = staging + ew * 2 * Y_BOX_BYTES;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint8_t* box = wstage + (c & 1) * Y_BOX_BYTES;
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<float4*>(box + lane * 128 + ((i ^ (lane & 7)) * 16)) =
                  make_float4(acc[c * 32 + 4 * i], acc[c * 32 + 4 * i + 1], acc[c * 32 + 4 * i + 2],
                              acc[c * 32 + 4 * i + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(ym, box, col0 + c * 32, ytop);
              bulk_commit();
            }
          }
        } else if (valid) {
          float* yrow = static_cast<float*>(tl.shared ? a.y_shared : a.y_perm) + yrow_at * a.d;
          float4* dst = reinterpret_cast<float4*>(yrow + col0);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        }
      }
    }
    if (PHASE == 2 && lane == 0) bulk_wait_all();   // outputs written before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// 2-D row-major FP32 tensor stored in 32 x 32 boxes with the 128-byte swizzle.
// 2-D row-major bf16 tensor stored in 32 x 64 boxes (128-byte rows) with the
// 128-byte swizzle.
inline int make_tmap_ybf(CUtensorMap* m, const uint16_t* base, uint64_t rows, uint64_t cols) {
  return make_tmap_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, Y_BOX, 2 * Y_BOX);
}

inline int make_tmap_y(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols) {
  return make_tmap_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, cols, Y_BOX, Y_BOX);
}

}  // namespace gg
}  // namespace moe

// H codes, H scales (from the next 256-byte boundary), then two int32 tile
// counters (one per launch, from the next 256-byte boundary)
static size_t counters_offset(size_t rows, int I) {
  return moe::gg::align256(moe::gg::align256(rows * I) + rows * (I / 128) * sizeof(float));
}

extern "C" size_t moe_grouped_gemm_fp8_rows_workspace(int P, int T, int d, int I) {
  (void)d;
  if (T <= 0 || P < 0 || I <= 0) return 0;
  const size_t rows = static_cast<size_t>(P) + T;
  return counters_offset(rows, I) + 2 * sizeof(int);
}

extern "C" size_t moe_grouped_gemm_fp8_workspace(int T, int K_r, int d, int I) {
  if (T <= 0 || K_r <= 0 || I <= 0) return 0;
  const long long P = static_cast<long long>(T) * K_r;
  if (P > (1LL << 31) - 1) return 0;
  return moe_grouped_gemm_fp8_rows_workspace(static_cast<int>(P), T, d, I);
}

// narrow tiles need the tile's [kb][token] activation-scale table to fit
// shared memory
static bool narrow_enabled(int d, int I) {
  return d / moe::gg::BK <= moe::gg::MAX_KB_N1 && I / moe::gg::BK <= moe::gg::MAX_KB_N2;
}

extern "C" int moe_grouped_gemm_fp8_launches(int d, int I) {
  if (d <= 0 || I <= 0) return -1;
  return 2;
}

// Both entry points: the routed rows come from xq_perm/xs_perm, or (sorted_token
// non-null) straight from xq/xs at the tokens sorted_token lists.
static int grouped_gemm(const uint8_t* xq_perm, const float* xs_perm, const int32_t* sorted_token,
                        const int32_t* offsets, int N_r, long long P, const uint8_t* xq, const float* xs, int T,
                        const uint8_t* w_gate, const uint8_t* w_up, const uint8_t* w_down, const float* s_gate,
                        const float* s_up, const float* s_down, int d, int I, uint16_t* y_perm, uint16_t* y_shared,
                        void* workspace, size_t ws_bytes, void* stream) {
  using namespace moe;
  using namespace moe::gg;
  MOE_CHECK_ARG(N_r >= 1 && P >= 0 && T >= 0 && d > 0 && I > 0);
  MOE_CHECK_SUPPORTED(N_r + 1 <= MAX_GROUPS && d % 256 == 0 && I % 128 == 0);
  MOE_CHECK_SUPPORTED(P + T < (1LL << 31) && static_cast<long long>(N_r + 1) * (d > I ? d : I) < (1LL << 31));
  if (T == 0) return MOE_OK;   // the shared expert's rows define the call (T = 0: nothing to do)
  const bool gather = sorted_token != nullptr;
  MOE_CHECK_ARG((gather || (xq_perm && xs_perm)) && offsets && xq && xs && w_gate && w_up && w_down && s_gate &&
                s_up && s_down && y_perm && y_shared && workspace);
  MOE_CHECK_ARG(ws_bytes >= moe_grouped_gemm_fp8_rows_workspace(static_cast<int>(P), T, d, I));
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(workspace) % 256 == 0 && reinterpret_cast<uintptr_t>(y_perm) % 16 == 0 &&
                reinterpret_cast<uintptr_t>(y_shared) % 16 == 0);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  cudaStream_t s = as_stream(stream);

  const long long rowsH = P + T;
  uint8_t* H = static_cast<uint8_t*>(workspace);
  float* Hs = reinterpret_cast<float*>(H + align256(static_cast<size_t>(rowsH) * I));

  CUtensorMap tmA, tmX, tmXg, tmWg, tmWu, tmH, tmWd, tmY, tmYs;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (int st = make_tmap_2d(&tmX, xq, U8, 1, T, d, BM, BK)) return st;
  if (gather) {
    // one-row boxes of xq for the four-row gathers; tmA is then unused
    if (int st = make_tmap_2d(&tmXg, xq, U8, 1, T, d, 1, BK)) return st;
    tmA = tmX;
  } else if (P == 0) {   // no routed rows: no tile reads tmA
    tmA = tmX;
    tmXg = tmX;
  } else {
    if (int st = make_tmap_2d(&tmA, xq_perm, U8, 1, P, d, BM, BK)) return st;
    tmXg = tmX;
  }
  if (int st = make_tmap_2d(&tmWg, w_gate, U8, 1, static_cast<uint64_t>(N_r + 1) * I, d, 128, BK)) return st;
  if (int st = make_tmap_2d(&tmWu, w_up, U8, 1, static_cast<uint64_t>(N_r + 1) * I, d, 128, BK)) return st;
  if (int st = make_tmap_2d(&tmH, H, U8, 1, rowsH, I, BM, BK)) return st;
  if (int st = make_tmap_2d(&tmWd, w_down, U8, 1, static_cast<uint64_t>(N_r + 1) * d, I, BN, BK)) return st;
  if (int st = make_tmap_ybf(&tmYs, y_shared, T, d)) return st;
  if (P > 0) {
    if (int st = make_tmap_ybf(&tmY, y_perm, P, d)) return st;
  } else {
    tmY = tmYs;
  }
  // Narrow tiles only when the average routed group has at most 64 rows
  // (decode-like batches). With larger groups the few small ones gain little
  // (an N <= 64 MMA costs about as much as an N = 256 one) and their slower
  // tiles put the CTAs out of step, so that tiles sharing weights and
  // activation rows no longer meet in L2 (measured with a static round-robin
  // schedule at T = 8192 with 39 groups of <= 64 rows: +4.2 GB of DRAM reads).
  const bool narrow = narrow_enabled(d, I) && P <= static_cast<long long>(NMAX) * N_r;

  Args args{};
  args.offsets = offsets;
  args.N_r = N_r;
  args.T = T;
  args.P = static_cast<int>(P);
  args.d = d;
  args.I = I;
  args.xs_perm = xs_perm;
  args.xs = xs;
  args.s_gate = s_gate;
  args.s_up = s_up;
  args.s_down = s_down;
  args.H = H;
  args.Hs = Hs;
  args.y_perm = y_perm;
  args.y_shared = y_shared;
  args.y_bf16 = 1;
  args.narrow_max = narrow ? NMAX : 0;
  args.sorted_token = sorted_token;
  int* counters = reinterpret_cast<int*>(H + counters_offset(static_cast<size_t>(rowsH), I));
  if (int st = cuda_status(cudaMemsetAsync(counters, 0, 2 * sizeof(int), s), "grouped GEMM: tile counters"))
    return st;

  // upper bound on row tiles: every non-empty routed group wastes < 1 tile
  const long long m_tiles = (P + BM - 1) / BM + (P < N_r ? P : N_r) + (T + BM - 1) / BM;
  const long long t1 = m_tiles * (I / 128), t2 = m_tiles * (d / BN);
  const int g1 = static_cast<int>(t1 < di.sm_count ? t1 : di.sm_count);
  const int g2 = static_cast<int>(t2 < di.sm_count ? t2 : di.sm_count);

  auto k1 = grouped_gemm_kernel<1>;
  auto k2 = grouped_gemm_kernel<2>;
  constexpr size_t sm1 = smem_bytes<1>(), sm2 = smem_bytes<2>();
  if (int st = cuda_status(cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm1)),
                           "smem attribute (gate/up)"))
    return st;
  if (int st = cuda_status(cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm2)),
                           "smem attribute (down)"))
    return st;
  args.tile_counter = counters;
  k1<<<g1, THREADS, sm1, s>>>(tmA, tmX, tmWg, tmWu, tmY, tmYs, tmXg, args);
  if (int st = launch_status("grouped GEMM launch (gate/up)")) return st;
  args.tile_counter = counters + 1;
  k2<<<g2, THREADS, sm2, s>>>(tmH, tmH, tmWd, tmWd, tmY, tmYs, tmXg, args);
  if (int st = launch_status("grouped GEMM launch (down)")) return st;
  return MOE_OK;
}

extern "C" int moe_grouped_gemm_fp8(const uint8_t* xq_perm, const float* xs_perm, const int32_t* offsets,
                                    int N_r, int K_r, const uint8_t* xq, const float* xs, int T,
                                    const uint8_t* w_gate, const uint8_t* w_up, const uint8_t* w_down,
                                    const float* s_gate, const float* s_up, const float* s_down, int d,
                                    int I, uint16_t* y_perm, uint16_t* y_shared, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (K_r < 1) return MOE_ERR_INVALID_ARG;
  return grouped_gemm(xq_perm, xs_perm, nullptr, offsets, N_r, static_cast<long long>(T) * K_r, xq, xs, T, w_gate,
                      w_up, w_down, s_gate, s_up, s_down, d, I, y_perm, y_shared, workspace, ws_bytes, stream);
}

extern "C" int moe_grouped_gemm_fp8_rows(const uint8_t* xq_perm, const float* xs_perm, const int32_t* offsets,
                                         int N_groups, int P, const uint8_t* xq, const float* xs, int T,
                                         const uint8_t* w_gate, const uint8_t* w_up, const uint8_t* w_down,
                                         const float* s_gate, const float* s_up, const float* s_down, int d, int I,
                                         uint16_t* y_perm, uint16_t* y_shared, void* workspace, size_t ws_bytes,
                                         void* stream) {
  if (P < 0) return MOE_ERR_INVALID_ARG;
  return grouped_gemm(xq_perm, xs_perm, nullptr, offsets, N_groups, P, xq, xs, T, w_gate, w_up, w_down, s_gate, s_up,
                      s_down, d, I, y_perm, y_shared, workspace, ws_bytes, stream);
}

extern "C" int moe_grouped_gemm_fp8_gather(const int32_t* sorted_token, const int32_t* offsets, int N_r, int K_r,
                                           const uint8_t* xq, const float* xs, int T, const uint8_t* w_gate,
                                           const uint8_t* w_up, const uint8_t* w_down, const float* s_gate,
                                           const float* s_up, const float* s_down, int d, int I, uint16_t* y_perm,
                                           uint16_t* y_shared, void* workspace, size_t ws_bytes, void* stream) {
  // a null sorted_token falls to the materialised-rows check (INVALID_ARG)
  if (K_r < 1) return MOE_ERR_INVALID_ARG;
  return grouped_gemm(nullptr, nullptr, sorted_token, offsets, N_r, static_cast<long long>(T) * K_r, xq, xs, T,
                      w_gate, w_up, w_down, s_gate, s_up, s_down, d, I, y_perm, y_shared, workspace, ws_bytes,
                      stream);
}

// A grouped scaled GEMM on the down-projection kernel: C = A B_g^T with A in
// the activation role (1x128 tiles along K) and B in the weight role (128x128
// blocks), the same FP32 promotion per 128-wide K block. The backward's
// products are of this form (dgrad with transposed weights; wgrad with one
// group whose rows are features and whose K is the expert's tokens).
extern "C" size_t moe_grouped_scaled_gemm_fp8_workspace(void) { return 256; }

extern "C" int moe_grouped_scaled_gemm_fp8(const uint8_t* a, const float* a_s, const int32_t* offsets, int N_groups,
                                           int P, int T, const uint8_t* b, const float* b_s, int K, int N, float* c,
                                           void* workspace, size_t ws_bytes, void* stream) {
  using namespace moe;
  using namespace moe::gg;
  MOE_CHECK_ARG(N_groups >= 0 && P >= 0 && T >= 1 && K > 0 && N > 0);
  MOE_CHECK_SUPPORTED(N_groups + 1 <= MAX_GROUPS && K % BK == 0 && N % BN == 0);
  MOE_CHECK_SUPPORTED(static_cast<long long>(P) + T < (1LL << 31) &&
                      static_cast<long long>(N_groups + 1) * N < (1LL << 31));
  MOE_CHECK_ARG(a && a_s && offsets && b && b_s && c && workspace);
  MOE_CHECK_ARG(ws_bytes >= moe_grouped_scaled_gemm_fp8_workspace());
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(workspace) % 16 == 0 && reinterpret_cast<uintptr_t>(c) % 16 == 0);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  cudaStream_t s = as_stream(stream);
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap tmA, tmB, tmC, tmCs;
  if (int st = make_tmap_2d(&tmA, a, U8, 1, static_cast<uint64_t>(P) + T, K, BM, BK)) return st;
  if (int st = make_tmap_2d(&tmB, b, U8, 1, static_cast<uint64_t>(N_groups + 1) * N, K, BN, BK)) return st;
  float* c_sh = c + static_cast<size_t>(P) * N;
  if (int st = make_tmap_y(&tmCs, c_sh, T, N)) return st;
  if (P > 0) {
    if (int st = make_tmap_y(&tmC, c, P, N)) return st;
  } else {
    tmC = tmCs;
  }
  Args args{};
  args.offsets = offsets;
  args.N_r = N_groups;
  args.T = T;
  args.P = P;
  args.d = N;          // the down kernel's output width
  args.I = K;          // and its contraction
  args.Hs = const_cast<float*>(a_s);
  args.s_down = b_s;
  args.y_perm = c;
  args.y_shared = c_sh;
  args.narrow_max = 0;
  args.sorted_token = nullptr;
  args.tile_counter = static_cast<int*>(workspace);
  if (int st = cuda_status(cudaMemsetAsync(workspace, 0, sizeof(int), s), "scaled GEMM: tile counter")) return st;
  const long long m_tiles = (P + BM - 1) / BM + (P < N_groups ? P : N_groups) + (T + BM - 1) / BM;
  const long long tiles = m_tiles * (N / BN);
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  auto k2 = grouped_gemm_kernel<2>;
  constexpr size_t sm2 = smem_bytes<2>();
  if (int st = cuda_status(cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm2)),
                           "smem attribute (scaled GEMM)"))
    return st;
  k2<<<grid, THREADS, sm2, s>>>(tmA, tmA, tmB, tmB, tmC, tmCs, tmA, args);
  return launch_status("scaled GEMM launch");
}

// K-grouped scaled GEMM on the same kernel: per group g,
// C_g = A[:, K_g] B[:, K_g]^T over the group's own K range K_g =
// kofs[g]..kofs[g+1]. The backward's weight gradients have this form: an
// expert's gradient contracts over that expert's tokens.
extern "C" size_t moe_kgrouped_gemm_fp8_workspace(void) { return 256; }

extern "C" int moe_kgrouped_gemm_fp8(const uint8_t* a, const float* a_s, const uint8_t* b, const float* b_s,
                                     const int32_t* kofs, int G, int M, int N, int K_total, float* c,
                                     void* workspace, size_t ws_bytes, void* stream) {
  using namespace moe;
  using namespace moe::gg;
  MOE_CHECK_ARG(G >= 1 && M >= 0 && N >= 0 && K_total >= 0);
  MOE_CHECK_SUPPORTED(G <= MAX_GROUPS - 1 && M % BM == 0 && N % BN == 0 && K_total % BK == 0);
  MOE_CHECK_SUPPORTED(static_cast<long long>(G) * M < (1LL << 31) && K_total < (1 << 30));
  if (M == 0 || N == 0) return MOE_OK;
  MOE_CHECK_ARG(c && workspace && ws_bytes >= moe_kgrouped_gemm_fp8_workspace());
  MOE_CHECK_ARG(reinterpret_cast<uintptr_t>(workspace) % 16 == 0 && reinterpret_cast<uintptr_t>(c) % 16 == 0);
  cudaStream_t s = as_stream(stream);
  if (K_total == 0)   // every group is empty: the products are zero
    return cuda_status(cudaMemsetAsync(c, 0, static_cast<size_t>(G) * M * N * sizeof(float), s),
                       "K-grouped GEMM: zero output");
  MOE_CHECK_ARG(a && a_s && b && b_s && kofs);
  DeviceInfo di;
  if (int st = device_info(&di)) return st;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap tmA, tmB, tmC;
  if (int st = make_tmap_2d(&tmA, a, U8, 1, M, K_total, BM, BK)) return st;
  if (int st = make_tmap_2d(&tmB, b, U8, 1, N, K_total, BN, BK)) return st;
  if (int st = make_tmap_y(&tmC, c, static_cast<uint64_t>(G) * M, N)) return st;
  Args args{};
  args.offsets = kofs;
  args.N_r = G - 1;
  args.T = M;
  args.P = 0;
  args.d = N;          // the down kernel's output width
  args.I = K_total;    // its contraction (all groups' K ranges)
  args.Hs = const_cast<float*>(a_s);
  args.s_down = b_s;
  args.y_perm = c;
  args.y_shared = c;
  args.narrow_max = 0;
  args.sorted_token = nullptr;
  args.kgrouped = 1;
  args.tile_counter = static_cast<int*>(workspace);
  if (int st = cuda_status(cudaMemsetAsync(workspace, 0, sizeof(int), s), "K-grouped GEMM: tile counter")) return st;
  const long long tiles = static_cast<long long>(G) * (M / BM) * (N / BN);
  const int grid = static_cast<int>(tiles < di.sm_count ? tiles : di.sm_count);
  auto k2 = grouped_gemm_kernel<2>;
  constexpr size_t sm2 = smem_bytes<2>();
  if (int st = cuda_status(cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm2)),
                           "smem attribute (K-grouped GEMM)"))
    return st;
  k2<<<grid, THREADS, sm2, s>>>(tmA, tmA, tmB, tmB, tmC, tmC, tmA, args);
  return launch_status("K-grouped GEMM launch");
}
