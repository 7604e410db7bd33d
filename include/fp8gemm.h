/*
 * fp8gemm.h -- C ABI of the fine-grained-scaled FP8 GEMM library for B200
 * (sm_100a).
 *
 * The operation (all three entry points):
 *
 *   D[m,n] = bf16_rne( sum_{kb} ( sum_{k = 128kb}^{128kb+127} A[m,k] * B[n,k] )
 *                               * sa[m,kb] * sb[n/128,kb] )
 *
 * A and B are FP8 e4m3 ("fn": bias 7, no infinities, max 448).  A carries one
 * FP32 scale per 1x128 group of a row; B carries one FP32 scale per 128x128
 * block.  This is the fine-grained scaling of DeepSeek-V3 (GeekNews, "DeepSeek,
 * DeepGEMM 오픈소스 공개", topic body, first bullet).  Each 128-wide K-block
 * partial is formed by the tensor cores and then promoted to an FP32
 * accumulator on the CUDA cores (same page, fifth bullet).  "NT": both operands
 * are K-major, so B is the transposed weight, and converting and transposing
 * inputs is the caller's job (kakushin.no, "Hvorfor FP8 og FP4 er
 * interessant").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers on the current device.  They are
 *    owned by the caller; the library neither allocates nor frees them.
 *  - Layouts are dense and row-major:
 *      A  [M, K] uint8 e4m3 codes, row pitch K bytes
 *      B  [N, K] uint8 e4m3 codes, row pitch K bytes
 *      sa [KB][ld_sa] float: sa[kb*ld_sa + m] scales A[m, 128kb .. 128kb+127]
 *         ("MN-major": one K-block's scales for consecutive rows are adjacent)
 *      sb [NB][KB] float: sb[nb*KB + kb] scales B[128nb .. +127, 128kb .. +127]
 *      D  [M, N] bf16 (bit patterns), row pitch N elements
 *    where KB = K/128 and NB = ceil(N/128).  If N % 128 != 0, the last scale
 *    block covers the remaining N % 128 rows.
 *  - Requirements (otherwise FP8G_ERR_INVALID_ARG / FP8G_ERR_MISALIGNED):
 *      K > 0, K % 128 == 0, K <= 65536; M, N >= 0; N % 8 == 0;
 *      ld_sa >= M (Mmax for the masked call) and ld_sa % 4 == 0;
 *      A, B, sa, D 16-byte aligned; sb, m_indices, masked_m 4-byte aligned.
 *    M == 0 or N == 0 (or G == 0) is a no-op that returns FP8G_OK.
 *  - The call enqueues kernels on `stream` and returns without waiting; D is
 *    complete when the stream reaches that point.  fp8_gemm_nt and the two
 *    grouped calls never read device memory on the host, so they can be
 *    captured in a CUDA graph.  The one exception to "never waits": see
 *    fp8_gemm_nt's workspace below.
 *  - Errors found on the host come back as the return value; nothing is
 *    launched then.  Errors found by the kernel (a bad m_indices entry, a
 *    masked_m above Mmax, a pipeline wait that timed out) are recorded in a
 *    per-device error word.  Read it with fp8g_get_device_error().  After a
 *    timeout the outputs of the calls since the word was last cleared are
 *    undefined (some CTAs gave up part-way).
 *  - The calls are thread-safe with respect to one another.
 *  - Needs a compute capability 10.0 device (B200); otherwise
 *    FP8G_ERR_UNSUPPORTED.
 */
#ifndef FP8GEMM_H
#define FP8GEMM_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fp8g_status {
    FP8G_OK = 0,
    FP8G_ERR_INVALID_ARG = 1,   /* null pointer, bad size, K % 128 != 0, ... */
    FP8G_ERR_MISALIGNED = 2,    /* pointer or pitch alignment not met */
    FP8G_ERR_UNSUPPORTED = 3,   /* device is not sm_100, or no kernel variant fits */
    FP8G_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (launch, attribute, ...) */
    FP8G_ERR_DEVICE = 5         /* fp8g_get_device_error found a recorded device-side error */
};

/* Device-side error word bits (fp8g_get_device_error). */
#define FP8G_DEVERR_TIMEOUT       0x1u  /* a pipeline wait gave up; outputs of that call are invalid */
#define FP8G_DEVERR_BAD_M_INDEX   0x2u  /* contiguous: m_indices entry >= G (block skipped) */
#define FP8G_DEVERR_MASKED_OVER   0x4u  /* masked: masked_m[g] > Mmax (clamped to Mmax) */
#define FP8G_DEVERR_BAD_EXPERT    0x8u  /* MoE dispatch: an expert id >= G or < -1 (row dropped) */

/*
 * Dense NT GEMM (GeekNews page, "일반 GEMM 성능 (Dense 모델)").
 *   A [M,K], sa [K/128][ld_sa], B [N,K], sb [ceil(N/128)][K/128], D [M,N].
 * Every element of D is written.
 * Decode shapes (M <= 64) split K over several CTAs per tile.  The first such
 * call on a device allocates a split-K workspace of about 4.7 MB (kept until
 * the process exits) and synchronises the device once.  If that first call
 * happens while `stream` is being captured, nothing is allocated and the call
 * uses a split-K kernel without a workspace (same results).  Callers that
 * cannot allocate at all use fp8_gemm_nt_no_alloc.
 */
int fp8_gemm_nt(const uint8_t *A, const float *sa, int ld_sa,
                const uint8_t *B, const float *sb,
                uint16_t *D, int M, int N, int K, cudaStream_t stream);

/*
 * M-grouped contiguous GEMM for MoE prefill/training (GeekNews page,
 * "연속된(contiguous) 레이아웃의 그룹화 GEMM": rows grouped along M, N and K shared).
 * The experts' row segments are concatenated along M.  Each segment is padded
 * to a multiple of 128 rows, so every 128-row block belongs to one expert.
 *   A [M,K] with M % 128 == 0, sa [K/128][ld_sa],
 *   B [G,N,K], sb [G][ceil(N/128)][K/128], D [M,N],
 *   m_indices [M/128] int32 (device): expert of each 128-row block.  -1 means
 *   the block belongs to no expert; its D rows are left untouched.  Padding
 *   rows inside a block are computed with that block's expert.
 */
int m_grouped_fp8_gemm_nt_contiguous(const uint8_t *A, const float *sa, int ld_sa,
                                     const uint8_t *B, const float *sb, uint16_t *D,
                                     const int32_t *m_indices,
                                     int M, int N, int K, int G, cudaStream_t stream);

/*
 * M-grouped masked GEMM for MoE decode under CUDA graphs (GeekNews page,
 * "마스킹(masked) 레이아웃의 그룹화 GEMM": the host does not know how many
 * tokens each expert got, so a mask tensor tells the kernel how much work to
 * do).
 *   A [G,Mmax,K], sa [G][K/128][ld_sa], B [G,N,K], sb [G][ceil(N/128)][K/128],
 *   D [G,Mmax,N], masked_m [G] int32 (device, never read on the host).
 * Group g computes its first min(masked_m[g], Mmax) rows; rows at and beyond
 * that count are left untouched.  expected_m is a hint (the typical
 * masked_m) used only to pick a kernel variant; results do not depend on it.
 */
int m_grouped_fp8_gemm_nt_masked(const uint8_t *A, const float *sa, int ld_sa,
                                 const uint8_t *B, const float *sb, uint16_t *D,
                                 const int32_t *masked_m,
                                 int G, int Mmax, int N, int K, int expected_m,
                                 cudaStream_t stream);

/*
 * Dense NT GEMM that allocates no device memory (the method's pages have no
 * counterpart: this serves callers that cannot allocate).
 *
 * Same operation, layouts, requirements and errors as fp8_gemm_nt.  It exists
 * for callers that must not call cudaMalloc when they run a GEMM: an engine
 * that hands out all device memory from its own pool, or a runtime that
 * forbids allocation after start-up so that its footprint is fixed in
 * advance.  fp8_gemm_nt allocates a split-K workspace
 * (about 4.7 MB) on the first decode-shaped call of each device; this entry
 * point instead keeps its scratch (the split-K partial sums and two counters
 * per tile) in a fixed array of 5 MiB + 1.25 KiB inside the library, which
 * every GPU that loads the library holds until the process exits.
 *  - It always runs the split-K kernel for decode shapes: tiles of 128 rows of
 *    B by 64 rows of A, K split over several CTAs per tile.  A shape with more
 *    than 160 such tiles (ceil(N/128) * ceil(M/64)), or more tiles than the GPU
 *    has SMs, needs more scratch than the array holds and returns
 *    FP8G_ERR_UNSUPPORTED without launching anything.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - Every call enqueues a small memset of its counters and one kernel on
 *    `stream`; it calls no cudaMalloc, cudaFree or other allocating routine.
 *  - All calls share the one array: calls whose executions overlap on the
 *    GPU (on different streams, or on one stream without ordering between
 *    them) race on it and give wrong results.  Order such calls.
 *  - The CTAs of one tile add their partial sums inside the kernel, so they
 *    must all be resident at once.  On a GPU shared with other work that may
 *    not happen within the wait limit (1 s); the call then records
 *    FP8G_DEVERR_TIMEOUT and D is undefined.
 */
int fp8_gemm_nt_no_alloc(const uint8_t *A, const float *sa, int ld_sa,
                         const uint8_t *B, const float *sb,
                         uint16_t *D, int M, int N, int K, cudaStream_t stream);

/*
 * Host helper: converts A's scales from the row-major layout a quantiser
 * naturally produces, src[g][m][kb] (one row of KB scales per row of A), to
 * the library's MN-major layout, dst[g][kb][ld_sa] (dst[(g*KB + kb)*ld_sa + m]
 * = src[(g*rows + m)*KB + kb]).  Entries m in [rows, ld_sa) of dst are set to
 * zero.  The pages leave the scale layout open; they only say that the
 * fine-grained scales come with the inputs (GeekNews, "DeepSeek, DeepGEMM
 * 오픈소스 공개", topic body, first bullet) and that preparing inputs is the
 * caller's job (kakushin.no, "Hvorfor FP8 og FP4 er interessant").
 *   src, dst: HOST pointers owned by the caller, not overlapping;
 *             src holds G*rows*KB floats, dst G*KB*ld_sa floats.
 *   G >= 1 groups (1 for dense and contiguous, G for the masked layout),
 *   rows >= 0 (M, or Mmax for masked), KB = K/128 >= 1,
 *   ld_sa >= rows and ld_sa % 4 == 0 (the GEMM calls' requirement).
 * Returns FP8G_OK; FP8G_ERR_INVALID_ARG for a null pointer or a bad size,
 * FP8G_ERR_MISALIGNED if ld_sa % 4 != 0.  Touches no device and no CUDA API.
 */
int fp8g_sa_to_mn_major(const float *src, float *dst, int G, int rows, int KB, int ld_sa);

/*
 * FP8 quantisers: the step before the GEMM that the pages leave to the caller
 * (kakushin.no, "Hvorfor FP8 og FP4 er interessant": inputs must be converted
 * to FP8 by the user), at the GEMM's granularity (GeekNews, "DeepSeek,
 * DeepGEMM 오픈소스 공개", topic body, first bullet: fine-grained scaling).
 * For every group G of input values:
 *     scale = amax(|G|) / 448   in FP32 (448 = the largest finite e4m3 value;
 *                               scale = 1 when every value of G is zero)
 *     code  = e4m3 of the FP32 quotient x / scale, rounded to nearest even,
 *             saturating at +-448 (one IEEE FP32 division per element).
 * The outputs are the GEMM calls' inputs, in their layouts.  Inputs must be
 * finite.  x_dtype is FP8G_IN_BF16 (x holds bf16 bit patterns) or
 * FP8G_IN_F32.  All pointers are DEVICE pointers owned by the caller; x must
 * not overlap the outputs.  The call enqueues one kernel on `stream` and
 * returns without waiting; it reads no device memory on the host and
 * allocates nothing.  Errors: FP8G_ERR_INVALID_ARG (null pointer, bad size
 * or dtype), FP8G_ERR_MISALIGNED (x and q not 16-byte aligned, sa not
 * 16-byte or sb not 4-byte aligned, ld_sa % 4 != 0), FP8G_ERR_CUDA (launch
 * failed).  rows == 0 or N == 0 is a no-op.
 */
#define FP8G_IN_BF16 0
#define FP8G_IN_F32 1

/*
 * Activations, one scale per 1x128 group of a row:
 *   x [rows][K] (K % 128 == 0)  ->  q [rows][K] e4m3 codes,
 *   sa [K/128][ld_sa] float, sa[kb*ld_sa + r] = scale of x[r, 128kb..+127]
 *   (ld_sa >= rows, ld_sa % 4 == 0; entries past `rows` are not written).
 */
int fp8g_quantize_1x128(const void *x, int x_dtype, int rows, int K,
                        uint8_t *q, float *sa, int ld_sa, cudaStream_t stream);

/*
 * Weights, one scale per 128x128 block:
 *   x [N][K] (K % 128 == 0)  ->  q [N][K] e4m3 codes,
 *   sb [ceil(N/128)][K/128] float, sb[nb*KB + kb] = scale of the block of
 *   rows 128nb.. (fewer in the last block row when N % 128 != 0) and
 *   columns 128kb..+127.
 */
int fp8g_quantize_128x128(const void *x, int x_dtype, int N, int K,
                          uint8_t *q, float *sb, cudaStream_t stream);

/*
 * The expert pipeline around the contiguous grouped GEMM.  The pages describe
 * only the layout the GEMM consumes (GeekNews, "MoE 모델을 위한 그룹화 GEMM
 * 성능": rows of A grouped along M by expert, N and K shared, each expert's
 * segment a whole number of 128-row blocks); these two calls build it from a
 * router's output and bring the GEMM's rows back to their tokens:
 *
 *   x [T][K] token activations --fp8g_moe_dispatch--> A, sa, m_indices, pos
 *   --m_grouped_fp8_gemm_nt_contiguous(M = blocks*128)--> D [blocks*128][N]
 *   --fp8g_moe_combine--> out [T][N]
 *
 * Routed row r = t*topk + k is slot k of token t; expert[r] is its expert in
 * [0, G), or -1 if it is dropped.  Expert g's rows keep their order r and fill
 * a segment padded up to a multiple of 128 rows; the segments follow each
 * other in expert order from row 0; pos[r] is row r's row in A (-1 if
 * dropped).  m_indices[b] is the expert of block b, -1 for the unused blocks
 * after the last segment (the GEMM skips them).  Nothing is read back on the
 * host, so with a fixed `blocks` the three calls can be captured in one CUDA
 * graph.  All pointers are DEVICE pointers owned by the caller; the calls
 * enqueue kernels on `stream` and return without waiting.
 */

/* Bytes of workspace fp8g_moe_dispatch needs for R = T*topk routed rows and
 * G experts (4 * (ceil(R/1024)*G + 2G)); 0 for bad arguments. */
size_t fp8g_moe_dispatch_workspace_bytes(int R, int G);

/*
 * Dispatch: builds the contiguous layout and quantises each routed row's
 * token into it, per 1x128 group (as fp8g_quantize_1x128).
 *   x [T][K] (bf16 patterns or FP32, x_dtype), K % 128 == 0, K <= 65536;
 *   expert [T*topk] int32; 1 <= topk <= 16; 1 <= G <= 256;
 *   blocks >= ceil(T*topk/128) + G (room for any routing);
 *   outputs A [blocks*128][K] e4m3 codes, sa [K/128][ld_sa] (ld_sa >=
 *   blocks*128, ld_sa % 4 == 0), pos [T*topk], m_indices [blocks];
 *   workspace: >= fp8g_moe_dispatch_workspace_bytes(T*topk, G) bytes,
 *   4-byte aligned, overwritten.
 * Padding rows of every segment get zero codes and zero scales (their D rows
 * are zero); rows of unused blocks are not written.  An expert id out of
 * range drops the row and sets FP8G_DEVERR_BAD_EXPERT.
 * Errors: FP8G_ERR_INVALID_ARG (bad size, capacity or workspace, null
 * pointer), FP8G_ERR_MISALIGNED (x, A, sa not 16-byte aligned; ld_sa), and
 * FP8G_ERR_CUDA.
 */
int fp8g_moe_dispatch(const void *x, int x_dtype, int T, int K,
                      const int32_t *expert, int topk, int G, int blocks,
                      uint8_t *A, float *sa, int ld_sa, int32_t *pos, int32_t *m_indices,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Combine: out[t][n] = bf16_rne(acc), acc = sum over k of w[t*topk + k] *
 * D[pos[t*topk + k]][n], accumulated in FP32 in slot order with one fused
 * multiply-add per slot (acc starts at 0; slots with pos < 0 are skipped;
 * w == NULL means weights of 1).  D [*][N] and out [T][N] are bf16 patterns,
 * N % 8 == 0, both 16-byte aligned; 1 <= topk <= 16 (as for the dispatch).
 * With topk == 1 and w == NULL it returns the GEMM's rows to token order.
 * Errors: FP8G_ERR_INVALID_ARG (bad size or topk, null pointer),
 * FP8G_ERR_MISALIGNED, FP8G_ERR_CUDA.
 */
int fp8g_moe_combine(const uint16_t *D, int N, const int32_t *pos, const float *w,
                     int T, int topk, uint16_t *out, cudaStream_t stream);

/*
 * BF16 NT GEMM on the same pipeline, the other input format the pages list
 * next to FP8 (kakushin.no, "Hva gjør DeepGEMM?"):
 *   D[m,n] = bf16_rne( sum_k A[m,k] * B[n,k] )   with FP32 accumulation,
 *   A [M,K], B [N,K], D [M,N] bf16 bit patterns, row-major and dense.
 * Requirements: K > 0, K % 64 == 0, K <= 65536, M, N >= 0, N % 8 == 0;
 * A, B, D 16-byte aligned (FP8G_ERR_INVALID_ARG / FP8G_ERR_MISALIGNED
 * otherwise).  Same conventions as fp8_gemm_nt: device pointers owned by the
 * caller, one kernel enqueued on `stream`, nothing read on the host.
 */
int bf16_gemm_nt(const uint16_t *A, const uint16_t *B, uint16_t *D,
                 int M, int N, int K, cudaStream_t stream);

/*
 * Dense NT GEMM with power-of-two (UE8M0) scales on the block-scaled tensor
 * cores of the SM100 generation the pages list (kakushin.no, requirements
 * list: SM90 and SM100):
 *   D[m,n] = bf16( sum_kb ( sum_{k in kb} A[m,k] * B[n,k] )
 *                         * 2^(sfa[kb][m] - 127) * 2^(sfb[n/128][kb] - 127) )
 * with the same 1x128 (A) and 128x128 (B) granularity as fp8_gemm_nt, but
 * the scales are E8M0 bytes (2^(e-127); 255 would be NaN and must not occur)
 * applied inside the tensor core, and the whole K sum is accumulated there
 * in FP32 (no per-K-block promotion), so results differ from fp8_gemm_nt's
 * within the GEMM tolerance; integer-valued inputs whose sums stay below 2^24
 * in units of the smallest scale are exact.
 *   A [M,K] e4m3, sfa [K/128][ld_sf] bytes (ld_sf >= M, ld_sf % 4 == 0),
 *   B [N,K] e4m3, sfb [ceil(N/128)][K/128] bytes, D [M,N] bf16.
 * Requirements and conventions otherwise as fp8_gemm_nt.
 */
int fp8_gemm_nt_ue8m0(const uint8_t *A, const uint8_t *sfa, int ld_sf,
                      const uint8_t *B, const uint8_t *sfb,
                      uint16_t *D, int M, int N, int K, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char *fp8g_status_string(int status);

/*
 * Reads this library's device-side error word on `device` into *bits (the
 * FP8G_DEVERR_* flags of every call since the last clear).  If `clear` is
 * nonzero, it also resets the word.  Synchronises the device.  Returns
 * FP8G_OK if the word is zero, FP8G_ERR_DEVICE if it is not, and
 * FP8G_ERR_CUDA if the read itself failed.
 */
int fp8g_get_device_error(int device, uint32_t *bits, int clear);

/*
 * Tuning and testing: force the kernel variant that the next calls use.
 * Pass -1 to restore automatic selection.  Variants are listed by
 * fp8g_variant_name(i) for i = 0 .. fp8g_num_variants()-1.  A forced variant
 * that cannot run a given call makes that call return FP8G_ERR_UNSUPPORTED.
 * The setting is process-wide.
 */
int fp8g_set_variant_override(int variant);
int fp8g_num_variants(void);
const char *fp8g_variant_name(int variant);

/*
 * The variant that the last successful call on this thread launched, or -1.
 */
int fp8g_last_variant(void);

/* Library version, major*10000 + minor*100 + patch. */
int fp8g_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8GEMM_H */
