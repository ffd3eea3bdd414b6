/*
 * moe_fp8.h - C ABI of the DeepSeekMoE FP8 layer forward pass on B200 (sm_100a).
 *
 * The layer (one MoE FFN of DeepSeek-V3) computes, for every token t,
 *
 *   h'_t = u_t + FFN^(s)(u_t) + sum_{i=1..N_r} g_{i,t} FFN^(r)_i(u_t)
 *   s_{i,t} = Sigmoid(u_t . e_i)
 *   g'_{i,t} = s_{i,t} if s_{i,t} + b_i is among the K_r largest of {s_{j,t} + b_j}, else 0
 *   g_{i,t}  = g'_{i,t} / sum_j g'_{j,t}
 *   b_i <- b_i - gamma (expert i overloaded) / b_i + gamma (underloaded), gamma = 0.001
 *
 * as printed in "DeepSeek-V3 Teknik Raporu" (xyznot.com/tr/paper/2412.19437),
 * section "Yöntem", part 2 "Yardımcı Kayıpsız Dengelemeli DeepSeekMoE", and in
 * its French copy "DeepSeek-V3 Technical Report" (xyznot.com/fr), "Méthode" 2.
 * The expert FFNs run in FP8 E4M3 with one FP32 scale per 1x128 activation tile
 * and per 128x128 weight block, accumulating in FP32 with the scales applied at
 * every 128-wide K block (same pages, "Temel fikirler" / "Idées clés", FP8
 * bullet: "FP8 Karma Duyarlıklı Eğitim").
 *
 * Conventions for every call
 *   - All pointers are DEVICE pointers owned by the caller, unless a comment
 *     says otherwise. No call allocates memory, and no call synchronises the
 *     host, except moe_get_error.
 *   - `stream` is a cudaStream_t passed as void*; work is enqueued on it.
 *   - Tensors are dense and row-major. bf16 is passed as uint16_t bits.
 *     FP8 tensors are uint8 E4M3 codes.
 *   - Activation scales are FP32, row-major [rows][cols/128], one per 1x128
 *     tile. Weight scales are FP32 [rows/128][cols/128], one per 128x128 block.
 *   - Expert weights are stacked over N_r + 1 slots; slot N_r is the shared
 *     expert. W_gate and W_up are [N_r+1][I][d] and W_down is [N_r+1][d][I]
 *     (K-major: the reduction dimension is contiguous).
 *   - Every call returns a moe_status. Arguments are checked on the host before
 *     any launch. A device-side failure (a wait that timed out) is recorded in a
 *     device error word that moe_get_error reads.
 *   - Stateless: the routing bias b is caller-owned state.
 */
#ifndef MOE_FP8_H
#define MOE_FP8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, workspace too small */
  MOE_ERR_UNSUPPORTED = 2,   /* a size outside what the kernels handle (see each call) */
  MOE_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
  MOE_ERR_TIMEOUT = 4,       /* a device wait exceeded its limit (read by moe_get_error) */
  MOE_ERR_NO_DEVICE = 5      /* no sm_100 device is current */
} moe_status;

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(int status);

/* Library version, e.g. 200 for 0.2.0. 0.2.0: expert outputs (y_perm,
 * y_shared of moe_grouped_gemm_fp8 and its variants, the rows moe_combine
 * reads) are bf16; moe_combine_fp32, moe_kgrouped_gemm_fp8 and
 * moe_route_quant added; the transposed quantisers write [cols][Ktot]. */
MOE_API int moe_version(void);

/*
 * Text describing the last host-side failure of a call made by this thread
 * (which CUDA call failed and its error string). Static per-thread buffer;
 * empty if nothing has failed.
 */
MOE_API const char* moe_last_error_detail(void);

/*
 * moe_get_error: synchronises the device, then reads and clears the device
 * error word that kernels set when a bounded wait gave up.
 *   device_status (HOST pointer, out): MOE_OK or MOE_ERR_TIMEOUT.
 * Returns MOE_OK, or MOE_ERR_CUDA if synchronising failed.
 */
MOE_API int moe_get_error(int* device_status);

/*
 * moe_quant_1x128: activation quantisation, one FP32 scale per 1x128 tile
 * ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8 bullet: 1x128 tile-wise
 * activation scaling, E4M3).
 *   x      [rows][cols] bf16 (input)
 *   q      [rows][cols] E4M3 (output)
 *   scale  [rows][cols/128] FP32 (output)
 * Per tile: amax = max |x|, scale = fl32(amax / 448) (1 if that is zero),
 * q = E4M3 round-to-nearest-even, saturating, of fl32(x / scale).
 * cols must be a multiple of 128 (else MOE_ERR_UNSUPPORTED); rows may be 0.
 */
MOE_API int moe_quant_1x128(const uint16_t* x, int rows, int cols, uint8_t* q,
                    float* scale, void* stream);

/*
 * moe_quant_128x128: weight quantisation, one FP32 scale per 128x128 block
 * (same passage: 128x128 block-wise weight scaling). Same scale rule as above.
 *   w      [rows][cols] FP32 (input)
 *   q      [rows][cols] E4M3 (output)
 *   scale  [rows/128][cols/128] FP32 (output)
 * rows and cols must be multiples of 128.
 */
MOE_API int moe_quant_128x128(const float* w, int rows, int cols, uint8_t* q,
                      float* scale, void* stream);

/*
 * moe_route: the router ("DeepSeek-V3 Teknik Raporu", Yöntem 2: the
 * s_{i,t}, g'_{i,t} and g_{i,t} equations).
 *   u          [T][d] bf16 token activations
 *   e          [N_r][d] bf16 expert centroids
 *   b          [N_r] FP32 routing bias (only affects selection)
 *   scores_in  NULL, or [T][N_r] FP32 affinities to use instead of
 *              Sigmoid(u . e) (u and e are then not read and may be NULL)
 *   scores_out NULL, or [T][N_r] FP32: the affinities s_{i,t}
 *   topk_idx   [T][K_r] int32: selected experts, ordered by key s+b
 *              descending, equal keys by lower index first
 *   gates      [T][K_r] FP32: g = s_sel / sum(s_sel), in the same order
 * The logits u . e run on the tensor cores in BF16 with FP32 accumulation; the
 * affinity uses the hardware exponential and approximate division (relative error
 * ~1e-6); the key s + b is formed in FP32. With few 128-token tiles the launch
 * is a set of thread-block clusters (2..8 CTAs per tile) that split d and add
 * their partial logits in a fixed order, so results do not depend on the
 * schedule. Limits: 1 <= K_r <= 16, K_r <= N_r <= 256, d a multiple of 64.
 * Errors: MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED before any launch;
 * MOE_ERR_CUDA if the launch fails (moe_last_error_detail names the call).
 */
MOE_API int moe_route(const uint16_t* u, const uint16_t* e, const float* b,
              const float* scores_in, int T, int d, int N_r, int K_r,
              float* scores_out, int32_t* topk_idx, float* gates,
              void* stream);

/*
 * moe_route_quant: moe_route from u and e (no scores_in) and, in the same
 * kernel, moe_quant_1x128 of u ("DeepSeek-V3 Teknik Raporu", Temel
 * fikirler, FP8 bullet: activations in 1x128 tiles): the router's epilogue
 * quantises the u tiles it streams for the logits, so u is read once for
 * both steps.
 *   xq, xs   [T][d] E4M3 and [T][d/128] FP32 (out): bit for bit what
 *            moe_quant_1x128(u) writes
 * Other arguments, outputs and limits as moe_route, and d a multiple of 128.
 */
MOE_API int moe_route_quant(const uint16_t* u, const uint16_t* e, const float* b,
                    int T, int d, int N_r, int K_r, float* scores_out,
                    int32_t* topk_idx, float* gates, uint8_t* xq, float* xs,
                    void* stream);

/*
 * moe_permute_workspace: bytes of scratch moe_permute needs for T tokens and
 * N_r experts (two int32 tables of ceil(T/256) x N_r).
 */
MOE_API size_t moe_permute_workspace(int T, int N_r);

/*
 * moe_permute: groups the (token, expert) pairs by expert with a stable
 * counting sort (histogram, prefix sum, scatter): row p of the permuted
 * layout holds token sorted_token[p]; rows are ordered by expert, then token.
 * The pages group tokens per expert without printing how; this is the plain
 * stable reading.
 *   topk_idx     [T][K_r] int32, each row distinct experts in [0, N_r)
 *   xq, xs       NULL, or the token rows to move: [T][d] E4M3, [T][d/128] FP32
 *   counts       [N_r] int32 (out): rows per expert
 *   offsets      [N_r+1] int32 (out): exclusive prefix sum of counts
 *   sorted_token [T*K_r] int32 (out)
 *   inv          [T][K_r] int32 (out): row of the pair (t, k)
 *   xq_perm, xs_perm  NULL (when xq is NULL) or [T*K_r][d], [T*K_r][d/128] (out)
 *   workspace    device scratch of moe_permute_workspace(T, N_r) bytes
 * Limits: N_r <= 1024, K_r <= 16, d a multiple of 128.
 * An expert index outside [0, N_r) records MOE_ERR_INVALID_ARG in the device
 * error word (moe_get_error); its pair gets inv = -1 and no row, and the rows
 * that pair would have filled are left unwritten.
 */
MOE_API int moe_permute(const int32_t* topk_idx, int T, int K_r, int N_r,
                const uint8_t* xq, const float* xs, int d,
                int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                int32_t* inv, uint8_t* xq_perm, float* xs_perm,
                void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_permute_noalloc: moe_permute for callers that cannot allocate device
 * memory (no workspace argument). The pages have no counterpart: this is a
 * deployment variant, not a step of the method. Same arguments, outputs and
 * limits as moe_permute, minus workspace/ws_bytes. Its scratch is a static
 * 1 MiB device array inside the library, held by every GPU that loads the
 * library until the process exits.
 *   - Sizes whose scratch (moe_permute_workspace(T, N_r)) exceeds 1 MiB are
 *     rejected with MOE_ERR_UNSUPPORTED (moe_last_error_detail says why).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. The address is cached per device index for
 *     the life of the process: after cudaDeviceReset (or any teardown of the
 *     device's primary context) the cached address is stale, so a process
 *     that resets a device must not call moe_permute_noalloc on it again.
 *   - All calls share the array: calls that overlap on the GPU (different
 *     streams, or different host threads, on the same device) race and must
 *     be serialised by the caller. Nothing needs clearing between calls.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
MOE_API int moe_permute_noalloc(const int32_t* topk_idx, int T, int K_r, int N_r,
                        const uint8_t* xq, const float* xs, int d,
                        int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                        int32_t* inv, uint8_t* xq_perm, float* xs_perm,
                        void* stream);

/*
 * moe_grouped_gemm_fp8_workspace: bytes of scratch for the intermediate
 * H = requant(SwiGLU(...)) of P = T*K_r routed rows plus T shared rows:
 * (P + T) * I bytes of E4M3 and (P + T) * I/128 FP32 scales. After a call the
 * workspace holds H: the codes [P + T][I] at its start (routed rows in
 * xq_perm order, then the T shared rows), and the scales [P + T][I/128] from
 * the next 256-byte boundary; after them (again 256-byte aligned) two int32
 * tile counters, which each call zeroes on its stream before its launches.
 */
MOE_API size_t moe_grouped_gemm_fp8_workspace(int T, int K_r, int d, int I);

/*
 * moe_grouped_gemm_fp8_launches: number of kernel launches one
 * moe_grouped_gemm_fp8 call with these sizes makes on its stream (2: the
 * gate/up launch and the down launch). A host-side query; no device work.
 * The pages have no counterpart: it exists so that callers can account for
 * launches. Returns -1 for non-positive sizes.
 */
MOE_API int moe_grouped_gemm_fp8_launches(int d, int I);

/*
 * moe_grouped_gemm_fp8: every expert FFN of the layer on FP8 operands.
 * For routed expert i (rows offsets[i]..offsets[i+1] of xq_perm) and for the
 * shared expert (slot N_r, all T rows of xq):
 *   G = X W_gate^T, U = X W_up^T      (FP8 x FP8 -> FP32)
 *   A = silu(G) * U,  H = quant_1x128(A)
 *   Y = H W_down^T, summed in FP32 and stored rounded to bf16
 * Each product is sum over 128-wide K blocks kb of
 *   s_X[m,kb] * s_W[n/128,kb] * (X_kb . W_kb),
 * the block partial coming from the tensor cores and the scaling and the sum
 * in FP32 ("Temel fikirler", FP8 bullet: FP32 promotion every N_c = 128).
 *   xq_perm, xs_perm  [P][d] E4M3, [P][d/128] FP32, P = T*K_r
 *   offsets           [N_r+1] int32 (device) from moe_permute
 *   xq, xs            [T][d], [T][d/128]: the shared expert's input
 *   w_gate, w_up      [N_r+1][I][d] E4M3;  s_gate, s_up  [N_r+1][I/128][d/128]
 *   w_down            [N_r+1][d][I] E4M3;  s_down        [N_r+1][d/128][I/128]
 *   y_perm            [P][d] bf16 (out)    y_shared [T][d] bf16 (out)
 *                     each element the FP32 result rounded to nearest even
 *   workspace         moe_grouped_gemm_fp8_workspace(T, K_r, d, I) bytes
 * Limits: d a multiple of 256, I a multiple of 128, N_r <= 1024.
 */
MOE_API int moe_grouped_gemm_fp8(const uint8_t* xq_perm, const float* xs_perm,
                         const int32_t* offsets, int N_r, int K_r,
                         const uint8_t* xq, const float* xs, int T,
                         const uint8_t* w_gate, const uint8_t* w_up,
                         const uint8_t* w_down, const float* s_gate,
                         const float* s_up, const float* s_down, int d, int I,
                         uint16_t* y_perm, uint16_t* y_shared,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_grouped_gemm_fp8_gather: moe_grouped_gemm_fp8 with the permutation's row
 * movement fused into the GEMM's loads: the routed rows are read from xq/xs
 * at the tokens sorted_token lists (moe_permute called with xq = NULL), so
 * xq_perm and xs_perm are never written or read. Same products, scales,
 * outputs, workspace and limits as moe_grouped_gemm_fp8 (the FP8 operands of
 * each row are the same bytes, so the outputs are bit-identical to it).
 *   sorted_token  [T*K_r] int32 (device) from moe_permute; values in [0, T)
 * The A tiles of routed rows arrive as four-row TMA gathers of xq, one per
 * lane of the producer warp per K block.
 */
MOE_API int moe_grouped_gemm_fp8_gather(const int32_t* sorted_token,
                         const int32_t* offsets, int N_r, int K_r,
                         const uint8_t* xq, const float* xs, int T,
                         const uint8_t* w_gate, const uint8_t* w_up,
                         const uint8_t* w_down, const float* s_gate,
                         const float* s_up, const float* s_down, int d, int I,
                         uint16_t* y_perm, uint16_t* y_shared,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_grouped_gemm_fp8_rows_workspace / moe_grouped_gemm_fp8_rows: the grouped
 * GEMM with an explicit count P of routed rows in N_groups groups instead of
 * P = T * K_r; the shared expert runs on T rows of xq (slot N_groups). Used
 * where the routed rows are not this batch's T * K_r pairs: under expert
 * parallelism a GPU runs its local experts on the rows the other GPUs sent
 * it ("DeepSeek 알고 아는 척 좀 해보자 – 단편: 671B 파라미터의 괴물,
 * DeepSeek-V3", "학습 인프라 & 최적화": 64-way expert parallelism). Same
 * products, scales, layouts and limits as
 * moe_grouped_gemm_fp8 (weights stacked over N_groups + 1 slots); P may be 0
 * (then xq_perm, xs_perm and y_perm may be NULL); T must be >= 1.
 */
MOE_API size_t moe_grouped_gemm_fp8_rows_workspace(int P, int T, int d, int I);
MOE_API int moe_grouped_gemm_fp8_rows(const uint8_t* xq_perm, const float* xs_perm,
                         const int32_t* offsets, int N_groups, int P,
                         const uint8_t* xq, const float* xs, int T,
                         const uint8_t* w_gate, const uint8_t* w_up,
                         const uint8_t* w_down, const float* s_gate,
                         const float* s_up, const float* s_down, int d, int I,
                         uint16_t* y_perm, uint16_t* y_shared,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_group_of_rows: out[p] = g mod modulo for every row p of a grouped layout
 * (offsets[g] <= p < offsets[g+1], offsets [n_groups+1] int32 on the device,
 * n_rows = offsets[n_groups]). Under expert parallelism the rows a GPU
 * receives are grouped by (source GPU, local expert): with modulo = local
 * experts this yields each row's local expert. No counterpart on the pages
 * (row bookkeeping around the all-to-all they describe, "DeepSeek-V3 Teknik
 * Raporu", "Problem ve motivasyon" item 2).
 */
MOE_API int moe_group_of_rows(const int32_t* offsets, int n_groups, int modulo,
                      int n_rows, int32_t* out, void* stream);

/*
 * moe_gather_rows: dst row i = src row idx[i] for i < n; rows of row_bytes
 * bytes (a multiple of 4), src holds n_src rows; src and dst 4-byte aligned
 * (16-byte rows and alignment move in 16-byte words). An index outside [0, n_src) is skipped and recorded as
 * MOE_ERR_INVALID_ARG in the device error word. Puts expert outputs back into
 * the order the rows arrived in before they return to their GPUs. No
 * counterpart on the pages.
 */
MOE_API int moe_gather_rows(const void* src, int n_src, const int32_t* idx, int n,
                    int row_bytes, void* dst, void* stream);

/*
 * ---------------------------------------------------------------- backward
 * The expert FFN's backward in the same FP8 scheme ("DeepSeek-V3 Teknik
 * Raporu", Temel fikirler, FP8 bullet: training in FP8 with E4M3 on all
 * tensors, activations in 1x128 tiles, weights in 128x128 blocks; the pages
 * print no backward details). Every backward GEMM has E4M3 operands; the
 * operand in the activation role (its rows are the product's rows) has one
 * FP32 scale per 1x128 tile along the contraction, the other one per 128x128
 * block; the requantisation of the intermediate is a cast (its gradient passes
 * through). wgrad contracts over an expert's tokens, each group's tokens
 * zero-padded to a multiple of 128.
 */

/*
 * moe_grouped_scaled_gemm_fp8: C = A B_g^T on the grouped GEMM kernel, FP32
 * promotion per 128-wide K block.
 *   a, a_s     [P+T][K] E4M3 and [P+T][K/128] FP32 (1x128 tiles); rows
 *              offsets[g]..offsets[g+1] (g < N_groups, offsets[N_groups] = P)
 *              use B slot g, the last T rows slot N_groups
 *   offsets    [N_groups+1] int32 (device); N_groups may be 0 (one group)
 *   b, b_s     [N_groups+1][N][K] E4M3, [N_groups+1][N/128][K/128] FP32
 *   c          [P+T][N] FP32 (out)
 *   workspace  moe_grouped_scaled_gemm_fp8_workspace() bytes (a tile counter)
 * Limits: K a multiple of 128, N a multiple of 256, T >= 1.
 */
MOE_API size_t moe_grouped_scaled_gemm_fp8_workspace(void);
MOE_API int moe_grouped_scaled_gemm_fp8(const uint8_t* a, const float* a_s,
                         const int32_t* offsets, int N_groups, int P, int T,
                         const uint8_t* b, const float* b_s, int K, int N,
                         float* c, void* workspace, size_t ws_bytes, void* stream);

/*
 * moe_kgrouped_gemm_fp8: for each group g < G, over its own K range
 * K_g = kofs[g] .. kofs[g+1] (elements),
 *   C_g = A[:, K_g] B[:, K_g]^T     (C_g = c + g * M * N, [M][N] FP32)
 * with FP32 promotion per 128-wide K block, on the grouped GEMM kernel. The
 * backward's weight gradients have this form (each expert contracts over its
 * own tokens), and one launch covers every expert.
 *   a, a_s   [M][K_total] E4M3, [M][K_total/128] FP32 (1x128 tiles along K)
 *   b, b_s   [N][K_total] E4M3, [N/128][K_total/128] FP32 (128x128 blocks)
 *   kofs     [G+1] int32 (device): non-decreasing multiples of 128 within
 *            [0, K_total]; a group with an empty range gets C_g = 0. A range
 *            that breaks this records MOE_ERR_INVALID_ARG in the device
 *            error word and its C_g is written as zero.
 *   workspace  moe_kgrouped_gemm_fp8_workspace() bytes (a tile counter)
 * Limits: M a multiple of 128, N a multiple of 256, K_total a multiple of
 * 128, G <= 1024.
 */
MOE_API size_t moe_kgrouped_gemm_fp8_workspace(void);
MOE_API int moe_kgrouped_gemm_fp8(const uint8_t* a, const float* a_s, const uint8_t* b,
                          const float* b_s, const int32_t* kofs, int G, int M, int N,
                          int K_total, float* c, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * moe_swiglu_backward_quant: for rows r < R and columns i < I,
 *   dG = dH U silu'(G),  dU = dH silu(G),  silu'(x) = s(x)(1 + x(1 - s(x)))
 * with s the sigmoid, then [dG | dU] ([R][2I]) quantised in 1x128 tiles:
 * q [R][2I] E4M3, qs [R][2I/128] FP32. g, u, dh [R][I] FP32 (G and U are the
 * forward's pre-activations, recomputed). dgu [R][2I] FP32: the unquantised
 * [dG | dU] (NULL: not written). I a multiple of 128.
 */
MOE_API int moe_swiglu_backward_quant(const float* g, const float* u, const float* dh,
                              int R, int I, float* dgu, uint8_t* q, float* qs,
                              void* stream);

/*
 * moe_quant_1x128_t / moe_quant_128x128_t: wgrad's operands. The rows of x
 * (row stride ld elements; columns 0..cols-1 are used) form n_groups groups,
 * rows src_off[g]..src_off[g+1]. The output is the transpose q [cols][Ktot]
 * E4M3 with Ktot = dst_off[n_groups]: group g fills its columns
 * dst_off[g] .. dst_off[g+1] of every row, its rows rounded up to a multiple
 * of 128 (the extra columns are zeros). Both offset arrays are int32 on the
 * device; dst_off[g] are multiples of 128.
 *   moe_quant_1x128_t:   x FP32 (x_is_bf16 = 0) or BF16; one scale per 1x128
 *                        tile along the tokens: s [cols][Ktot/128]
 *   moe_quant_128x128_t: x E4M3 rows with 1x128 scales xs [rows][ld/128]
 *                        (the forward's FP8 activations), each value
 *                        dequantised (rounded once to FP32) and requantised in
 *                        128x128 blocks: s [cols/128][Ktot/128]
 * cols and Ktot multiples of 128. A 128-wide token block never spans two
 * groups, so every tile and block holds one expert's tokens.
 */
MOE_API int moe_quant_1x128_t(const void* x, int x_is_bf16, int ld, int cols,
                      const int32_t* src_off, const int32_t* dst_off, int n_groups,
                      int Ktot, uint8_t* q, float* s, void* stream);
MOE_API int moe_quant_128x128_t(const uint8_t* xq, const float* xs, int ld, int cols,
                        const int32_t* src_off, const int32_t* dst_off, int n_groups,
                        int Ktot, uint8_t* q, float* s, void* stream);

/*
 * moe_transpose: for b < batch, dst[b][j][dst_col + i] = src[b][i][j] with
 * src [batch][rows][cols] and dst [batch][cols][dst_ld]; elements of
 * elem_bytes = 1 (E4M3 codes) or 4 (FP32 scales). The weights' codes and
 * block scales for dgrad: a 128x128 block stays one block when transposed,
 * so the transposed weight is exact.
 */
MOE_API int moe_transpose(const void* src, int elem_bytes, int batch, int rows, int cols,
                  void* dst, int dst_ld, int dst_col, void* stream);

/*
 * moe_combine: h'_t = bf16(u_t + y_shared_t + sum_k g_{t,k} y_perm[inv[t][k]])
 * ("DeepSeek-V3 Teknik Raporu", Yöntem 2, the h'_t equation). The sum is FP32
 * in the fixed order u, shared, k = 0..K_r-1.
 *   u [T][d] bf16;  y_shared [T][d] bf16;  y_perm [T*K_r][d] bf16;  inv, gates [T][K_r]
 *   out [T][d] bf16 (may alias u)
 * d must be a multiple of 8.
 */
MOE_API int moe_combine(const uint16_t* u, const uint16_t* y_perm,
                const uint16_t* y_shared, const int32_t* inv,
                const float* gates, int T, int K_r, int d, uint16_t* out,
                void* stream);

/*
 * moe_combine_fp32: moe_combine with FP32 rows y_perm, y_shared (the
 * backward sums the FP32 input gradients of a token's rows with it, gates 1).
 */
MOE_API int moe_combine_fp32(const uint16_t* u, const float* y_perm,
                     const float* y_shared, const int32_t* inv,
                     const float* gates, int T, int K_r, int d, uint16_t* out,
                     void* stream);

/*
 * moe_bias_update: auxiliary-loss-free balancing ("DeepSeek-V3 Teknik
 * Raporu", Yöntem 2, last paragraph): b_i -= gamma when expert i is
 * overloaded, b_i += gamma when underloaded. Overloaded means
 * counts[i] * N_r > T * K_r (load above the mean); equal load leaves b_i.
 *   b                  [N_r] FP32, updated in place
 *   counts             [N_r] int32 from moe_permute
 *   max_over_mean_out  NULL or [1] FP32 (device): max_i counts[i] * N_r / (T*K_r)
 */
MOE_API int moe_bias_update(float* b, const int32_t* counts, int N_r, int T, int K_r,
                    float gamma, float* max_over_mean_out, void* stream);

/*
 * moe_debug_wait_timeout: launches one block that waits on a barrier nothing
 * ever signals, with a limit of timeout_us microseconds; the wait gives up and
 * records MOE_ERR_TIMEOUT in the device error word. Exists to test the
 * timeout path without hanging a GPU. 1 <= timeout_us <= 1000000.
 */
MOE_API int moe_debug_wait_timeout(int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FP8_H */
