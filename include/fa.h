/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa_b200.so).
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T + mask) V,      L_i = ln sum_j exp(scale * q_i . k_j + mask_ij)
 *
 * block by block with an online softmax, so the N x N score matrix never reaches
 * device memory.  The formula is the one the FlashAttention pages print
 * (FlashAttention (NL), "Problemen met standaard attention", with 1/sqrt(d_k) as the
 * usual scale); the tiling, the online softmax (running row maximum and running sum of
 * exponentials) and the single fused kernel are that page's "Tiling en blokgewijze
 * verwerking", "Online berekening van Softmax" and "Samensmelting van bewerkingen in een
 * CUDA-kernel"; the backward recomputes the probabilities from L instead of storing them
 * (memory-optimized flash attention page, "How it works").
 *
 * Conventions shared by every entry point
 *   Layout     Q, K, V, O, dO, dQ, dK, dV are contiguous bf16 arrays [B, H, N, d] (d fastest,
 *              row stride d elements, head stride N*d); L is contiguous fp32 [B, H, N].
 *              Self-attention: queries and keys have the same length N.
 *   Pointers   every array argument is a DEVICE pointer of the current CUDA device; the
 *              caller allocates, owns and frees all of them.  The library allocates no
 *              device memory and keeps no pointer after a call returns.
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *              Every call only enqueues work on that stream and returns; it never
 *              synchronises (fa_check_status excepted).
 *   Masks      causal = 1 keeps key j for query i iff j <= i.  window = W > 0 with
 *              causal = 1 also requires j >= i - W + 1 (one-sided band); with causal = 0
 *              it keeps |i - j| <= W - 1 (the local window on both sides).  Either band
 *              counts the diagonal, so W = 1 keeps only key i; window = 0 means no band.
 *              (The sparse-attention glossary, "Abgrenzung & Vergleiche", names sliding-
 *              window attention as a purely local window and fixes no convention.)  Keys
 *              j >= N never exist.  Every query keeps its diagonal, so no row is empty.
 *   Scale      applied inside: S = scale * Q K^T.  Must be finite and > 0.
 *   Errors     arguments are validated before anything is enqueued; a rejected call
 *              returns its FA_ERR_* code and touches no memory.  A failed launch returns
 *              FA_ERR_CUDA.  Kernel-side waits are bounded: one that runs out records a
 *              timeout in a device status word that fa_check_status() reports.
 *   Device     a compute-capability 10.0 GPU (B200, sm_100a); others give FA_ERR_DEVICE.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_EXPORT __attribute__((visibility("default")))
#else
#define FA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = 1,       /* a required pointer is NULL */
  FA_ERR_SHAPE = 2,      /* a size < 1, H not a multiple of H_kv, N_q > N_k, or beyond the launch limits */
  FA_ERR_HEADDIM = 3,    /* d is not 64, 128 or 256 */
  FA_ERR_ALIGN = 4,      /* a bf16 array is not 16-byte aligned, or L not 4-byte aligned */
  FA_ERR_MASK = 5,       /* causal not 0/1, or window < 0 */
  FA_ERR_WORKSPACE = 6,  /* workspace missing or smaller than fa_bwd_ / fa_decode_workspace_size */
  FA_ERR_CUDA = 7,       /* a CUDA runtime call or kernel launch failed */
  FA_ERR_DEVICE = 8,     /* the current device is not compute capability 10.0 */
  FA_ERR_TIMEOUT = 9,    /* a kernel-side wait ran out of time (reported by fa_check_status) */
  FA_ERR_SCALE = 10,     /* scale is not finite and > 0 */
  FA_ERR_NOALLOC_LIMIT = 11, /* fa_bwd_noalloc: fa_bwd_workspace_size(...) exceeds its 64 MiB scratch */
  FA_ERR_INTERNAL = 12,  /* a kernel found it could not run as built (reported by fa_check_status) */
  FA_ERR_PHASES = 13     /* fa_bwd_phases: phase mask outside 1..7 */
} fa_status;

/*
 * Forward pass.  Writes O (bf16 [B,H,N,d]) and L (fp32 [B,H,N], natural-log logsumexp of
 * the masked, scaled scores of each query row).  Reads q, k, v (bf16 [B,H,N,d]).
 * d must be 64, 128 or 256.  Extra device memory: none beyond O and L.  d = 256 runs a kernel of
 * its own (one 128-row query tile per CTA, 64-key K/V tiles).
 */
FA_EXPORT int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, int window, void* stream);

/*
 * Bytes of device workspace fa_bwd needs: 4 * B*H * Np * (d + 2) with Np = N rounded up to
 * a multiple of 128 (per row: D, L in log2 units, and a d-wide fp32 dQ accumulator).
 * Returns 0 when the shape itself is invalid.  O(N * d): no N x N buffer.
 */
FA_EXPORT size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass with recomputation.  From q, k, v, the forward's o and lse, and the output
 * gradient dO (bf16 [B,H,N,d]) it writes dQ, dK, dV (bf16 [B,H,N,d]): the gradients of
 * sum(O o dO).  Same mask, scale and shape arguments as the forward that produced o and lse.
 * `workspace` (device, caller-owned, 16-byte aligned, at least fa_bwd_workspace_size bytes)
 * is scratch: it is overwritten and may be reused once the call's work has completed on
 * `stream`.  Three kernels are enqueued: D = rowsum(dO o O) with a cleared accumulator, the
 * fused recompute kernel, and the dQ scaling.  d must be 64, 128 or 256; d = 256 runs a kernel of
 * its own (one CTA per 64-key tile and head-dim half).
 */
FA_EXPORT int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, int window,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * The backward pass split into its three phases, so that a caller can time or interleave
 * them.  `phases` is a mask of
 *   1  preprocess: D = rowsum(dO o O), L in log2 units and a cleared fp32 dQ accumulator,
 *      all in `workspace`;
 *   2  the recompute kernel: dK and dV written, dQ accumulated in `workspace`;
 *   4  finalise: dQ = scale * accumulator, written as bf16.
 * Calling it with 1, then 2, then 4 on one stream with the same arguments and workspace
 * does exactly what one fa_bwd call (mask 7) does.  Arguments, validation and errors are
 * fa_bwd's; a mask outside 1..7 gives FA_ERR_PHASES.
 */
FA_EXPORT int fa_bwd_phases(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                            int causal, int window, void* workspace, size_t workspace_bytes, int phases,
                            void* stream);

/*
 * Element strides of one bf16 array of logical shape [B, heads, N, d] whose d elements are
 * contiguous: element (b, h, n, c) is at b * b_stride + h * h_stride + n * n_stride + c.  The
 * packed layout [B, heads, N, d] is {heads*N*d, N*d, d}; [B, N, heads, d] (sequence-major) is
 * {N*heads*d, d, heads*d}.
 */
typedef struct fa_strides {
  long long b, h, n;
} fa_strides;

/*
 * Shared K/V heads (multi-query and grouped-query attention).  The FlashAttention (NL) page
 * lists Multi-Query Attention among what FlashAttention-2 supports ("Evolutie en verdere
 * ontwikkelingen"); here H query heads read H_kv K/V heads (H a multiple of H_kv; H_kv = 1 is
 * multi-query, H_kv = H is fa_fwd / fa_bwd), in contiguous groups: query head h reads K/V
 * head h / (H / H_kv).  q, o, dO, dq: bf16 [B,H,N,d]; k, v, dk, dv: bf16 [B,H_kv,N,d]; lse:
 * fp32 [B,H,N].  dk and dv are the sums over each K/V head's query heads.  Everything else
 * (masks, scale, ownership, errors, streams) is as for fa_fwd / fa_bwd; the workspace is
 * fa_bwd_workspace_size(B, H, N, d) bytes (it scales with the query heads), and `phases` is
 * as for fa_bwd_phases (7 = the whole backward).  FA_ERR_SHAPE also when H_kv < 1 or H is not
 * a multiple of H_kv.
 */
FA_EXPORT int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                         int N, int d, float scale, int causal, int window, void* stream);
FA_EXPORT int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
                         float scale, int causal, int window, void* workspace, size_t workspace_bytes,
                         int phases, void* stream);

/*
 * fa_fwd_gqa / fa_bwd_gqa on arrays with arbitrary strides (for instance the sequence-major
 * [B, N, H, d] layout of many frameworks) instead of packed ones.  `strides` (host memory)
 * holds one fa_strides per array: q, k, v, o for the forward (4 entries, or NULL for packed
 * arrays); q, k, v, o, dO, dq, dk, dv for the backward (8 entries, not NULL).  Every stride must
 * be a positive multiple of 8 elements (FA_ERR_ALIGN otherwise); strides that make an output
 * overlap itself are the caller's error.  lse stays packed fp32 [B, H, N].  The pages print no
 * layout: the strides only say where the same [B, heads, N, d] elements live.
 */
FA_EXPORT int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int H_kv, int N, int d, const fa_strides* strides, float scale, int causal, int window,
                             void* stream);
FA_EXPORT int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
                             const fa_strides* strides, float scale, int causal, int window, void* workspace,
                             size_t workspace_bytes, int phases, void* stream);

/*
 * Forward of a few new query rows over a longer key sequence: a generation step over a
 * key/value cache.  The FlashAttention (NL) page names engines for LLM inference that work on
 * the key/value cache during streaming generation ("Gespecialiseerde oplossingen": FlashInfer;
 * its references add FlashDecoding++); it prints no interface.  Reading: the N_q query rows are
 * the last N_q of the N_k key positions, so query row i stands at position N_k - N_q + i and
 * the masks of fa_fwd apply there (causal: keys j <= N_k - N_q + i; with a window W also
 * j >= N_k - N_q + i - W + 1; a window without causal keeps |j - (N_k - N_q + i)| <= W - 1).
 * N_q = N_k is the self-attention of fa_fwd_gqa.
 *
 *   q, o   bf16 [B, H, N_q, d];  k, v  bf16 [B, H_kv, N_k, d]  (H a multiple of H_kv; query
 *          head h reads K/V head h / (H / H_kv));  lse  fp32 [B, H, N_q], packed.
 *   strides  NULL for packed arrays, else 4 fa_strides (q, k, v, o) as for fa_fwd_strided.
 *   d      64, 128 or 256.
 *   workspace  device memory of at least fa_decode_workspace_size(...) bytes, 16-byte aligned,
 *          owned by the caller; it holds the per-split partial results (fp32).  When that size
 *          is 0 (the keys fit one split) workspace may be NULL.
 *
 * The keys are cut into splits that run on separate CTAs; a second kernel merges the splits'
 * partial outputs by their logsumexps.  How the problem is cut depends only on the arguments
 * of fa_decode_workspace_size, which returns 0 for an invalid problem.  Errors, scale, streams
 * and ownership are as for fa_fwd; FA_ERR_SHAPE also when N_q > N_k, FA_ERR_WORKSPACE when the
 * workspace is missing or short.
 */
FA_EXPORT size_t fa_decode_workspace_size(int B, int H, int H_kv, int N_q, int N_k, int d, int causal, int window);
FA_EXPORT int fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                            int N_q, int N_k, int d, const fa_strides* strides, float scale, int causal, int window,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_fwd_decode over an FP8 key/value cache.  The FlashAttention (NL) page says FlashAttention-3
 * supports FP8 ("Evolutie en verdere ontwikkelingen"), without a format; the reading is that
 * paper's E4M3 with one scale per tensor: K = k_scale * E4M3(k8), V = v_scale * E4M3(v8), where
 * E4M3 has 1 sign, 4 exponent (bias 7) and 3 mantissa bits, subnormals, no infinities, and
 * S.1111.111 as NaN (NaN codes give NaN results).
 *
 *   k8, v8   E4M3 codes, one byte each, [B, H_kv, N_k, d]; with `strides`, their strides count
 *            bytes and must be multiples of 16.
 *   k_scale, v_scale  finite and > 0 (FA_ERR_SCALE otherwise).
 *   everything else as for fa_fwd_decode (q, o bf16; lse fp32; the same workspace size,
 *   fa_decode_workspace_size).
 *
 * The kernels convert the codes to f16, which is exact, and run the products with f16 operands:
 * Q is rounded to f16 after clamping to +-65504, and P enters P V as f16.  k_scale multiplies
 * the softmax scale; v_scale multiplies O before it is rounded to bf16.
 */
FA_EXPORT int fa_fwd_decode_fp8kv(const void* q, const void* k8, const void* v8, float k_scale, float v_scale,
                                  void* o, float* lse, int B, int H, int H_kv, int N_q, int N_k, int d,
                                  const fa_strides* strides, float scale, int causal, int window, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * Forward on FP8 (E4M3) Q, K and V with one scale per tensor: Q = q_scale * E4M3(q8),
 * K = k_scale * E4M3(k8), V = v_scale * E4M3(vt8)^T; the FP8 forward the FlashAttention (NL)
 * page attributes to FlashAttention-3 ("Evolutie en verdere ontwikkelingen").  E4M3 as for
 * fa_fwd_decode_fp8kv.  Both products run on the tensor cores' 8-bit path (E4M3 x E4M3 -> fp32);
 * P is rounded to E4M3 before P V (O carries that rounding: relative 2^-4 per weight).
 *
 *   q8     E4M3 codes [B, H, N, d], packed;  k8  [B, H_kv, N, d], packed.
 *   vt8    V transposed: E4M3 codes [B, H_kv, d, N], packed (N contiguous), so that both operands
 *          of the 8-bit P V product are K-major.
 *   o, lse bf16 [B, H, N, d] and fp32 [B, H, N], packed.
 *   d must be 128 (FA_ERR_HEADDIM otherwise); N a multiple of 16 (FA_ERR_SHAPE); the scales
 *   finite and > 0 (FA_ERR_SCALE).  Masks, scale, errors and streams as for fa_fwd_gqa.
 *
 */
FA_EXPORT int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, float q_scale, float k_scale, float v_scale,
                         void* o, float* lse, int B, int H, int H_kv, int N, int d, float scale, int causal, int window,
                         void* stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_EXPORT const char* fa_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the device status word of the current
 * device.  Returns FA_ERR_INTERNAL if a kernel since the last check refused to run (its
 * dynamic shared memory was not 1 KB aligned), else FA_ERR_TIMEOUT if one gave up on a
 * bounded wait, FA_ERR_CUDA if the synchronisation failed, FA_OK otherwise.
 */
FA_EXPORT int fa_check_status(void* stream);

/*
 * Time limit, in nanoseconds, of every kernel-side wait launched after this call
 * (process-wide; default 4e9 = 4 s).  0 restores the default.
 */
FA_EXPORT void fa_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * Failure-detection self-test: enqueues one small kernel that waits on a barrier nothing
 * ever completes, under a limit of `limit_ns` nanoseconds (clamped to [1 us, 1 s]).  The
 * wait runs out, the kernel records a timeout and exits, and the next fa_check_status()
 * returns FA_ERR_TIMEOUT.  No memory is touched besides the status word.
 */
FA_EXPORT int fa_selftest_timeout(unsigned long long limit_ns, void* stream);

/*
 * Backward pass for callers that cannot allocate device memory.  The FlashAttention pages
 * have no counterpart of this entry point; it exists for code that may not call cudaMalloc
 * and has no allocator to ask: for example an operator running as a plugin inside a host
 * framework that owns all device memory, or a latency-critical service that forbids
 * allocation (which can synchronise the device) once it has started.
 *
 * Same arguments and results as fa_bwd, without the workspace: the scratch (D, L and the
 * fp32 dQ accumulator) lives in one 64 MiB array inside the library, which every GPU that
 * loads the library holds until the process exits.  Problems whose
 * fa_bwd_workspace_size(B, H, N, d) exceeds 64 MiB (67108864 bytes) are rejected with
 * FA_ERR_NOALLOC_LIMIT before anything is enqueued; for d = 128 that allows
 * B*H*ceil(N/128)*128 <= 129055 rows, e.g. 31 heads of N = 4096.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current), so make that first call before any stream capture begins.
 * The call itself allocates nothing (no cudaMalloc, cudaFree or allocating library call);
 * every scratch byte the kernels read is rewritten at the start of each call.  All calls
 * share the one array: two calls whose work overlaps on the GPU (different streams, or
 * several host threads) race on it and give wrong results -- serialise them.
 */
FA_EXPORT int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                             float scale, int causal, int window, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
