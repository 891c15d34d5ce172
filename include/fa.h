/*
 * exact IO-aware attention for NVIDIA B200 (sm_100a): the C ABI.
 *
 * The operation is exact scaled-dot-product attention, one head at a time,
 *     S = tau * Q K^T,  P = softmax(mask(S)) row by row,  O = dropout(P) V,
 * as defined in "FlashAttention 的第一原则" (reader.mx), section 2 (Q, K, V and O are N x d,
 * the N x N intermediates, optional mask and dropout) and section 3.2 (op order matmul, scale,
 * mask, softmax, dropout), and in "48 FlashAttention" (ml-canon), block "PyTorch FlashAttention
 * под капотом sdpa" (result identical to softmax(QK^T/sqrt(d)) V).  The forward computes it tile
 * by tile with an online softmax (same page, block "Tiling и online softmax"): the N x N scores
 * never reach device memory.  The backward recomputes each probability block from Q, K and the
 * saved per-row logsumexp (same page, block "Backward — тоже без N×N").
 *
 * Conventions for every entry point below.
 *  - Layouts: q, k, v, o, dO, dq, dk, dv are [B, H, N, d] row-major contiguous (d innermost);
 *    lse is [B, H, N] fp32, natural log, lse = m + ln(l) over the masked, scaled scores and
 *    the undropped probabilities.  key_lens is int32 [B] on the device, or NULL.
 *  - Masks: causal keeps key j <= query i (top-left aligned, self-attention: one N for
 *    queries and keys); key padding keeps j < key_lens[b] (keys only; every query row is
 *    computed).  A row with no allowed key gets O = 0, lse = -inf and zero gradients.
 *  - Dropout (0 <= dropout_p < 1): element (b, h, i, j) is kept when the counter hash
 *      ctr = ((b*H + h)*N + i)*N + j,  z = seed + (ctr + 1) * 0x9E3779B97F4A7C15 (mod 2^64),
 *      z = SplitMix64 output mix of z,  keep = (z >> 32) >= min(floor(p * 2^32), 2^32 - 1)
 *    holds; kept probabilities are multiplied by 1/(1 - p).  The backward must get the same
 *    (scale, causal, key_lens, dropout_p, seed) as the forward it differentiates.
 *  - Pointers are DEVICE pointers owned by the caller, 16-byte aligned; the library never
 *    allocates or frees device memory.  Outputs are overwritten, not accumulated.
 *  - scale (tau) must be finite and > 0 (1/sqrt(d) is the usual value).
 *  - bf16 entry points support d in {64, 128} (fa_fwd also d = 256), fa_fwd_f32 any 1 <= d <= 128;
 *    N >= 1 is arbitrary (tails are zero-filled by the tile loads and masked); B*H <= 65535.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  The return value reports argument validation and launch errors only.  Errors
 *    found on the device (a bounded wait that ran out) are reported by fa_check().
 *  - On a non-OK return, fa_get_error() describes the failure (thread-local string).
 */
#ifndef EXACT_IO_AWARE_FA_H
#define EXACT_IO_AWARE_FA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

/* The CUDA stream handle, as the CUDA runtime declares it (driver_types.h), so that this header
 * needs no CUDA include; a driver-API CUstream is the same type.  If the runtime header comes after
 * this one, the repeated typedef is legal C11 and C++. */
#ifndef __DRIVER_TYPES_H__
typedef struct CUstream_st* cudaStream_t;
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* a null or misaligned pointer, a size or parameter out of range */
  FA_ERR_UNSUPPORTED = 2,  /* a valid request this build does not implement (e.g. bf16 with d = 96) */
  FA_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed */
  FA_ERR_TIMEOUT = 4,      /* a kernel's bounded wait ran out; its outputs are undefined */
  FA_ERR_INTERNAL = 5      /* the device reported an inconsistent launch (e.g. shared memory alignment) */
} fa_status;

/* Forward, bf16 ("48 FlashAttention", block "Tiling и online softmax": tile by tile with a running
 * row max m and row sum l, O re-expressed when m moves; the operation of "FlashAttention 的第一原则",
 * section 2).  Writes o (bf16 [B,H,N,d]) and lse (fp32 [B,H,N]).  q, k, v: bf16 [B,H,N,d].
 * d in {64, 128, 256} (d = 256 has no backward).  One kernel launch. */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, float scale, int causal,
                 const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream);

/* Forward, fp32 throughout (CUDA-core FFMA, no TF32; the same online softmax), same semantics and
 * layouts with fp32 q, k, v, o.  Any head dimension 1 <= d <= 128.  One kernel launch. */
FA_API fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
                     int B, int H, int N, int d, float scale, int causal,
                     const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream);

/* Bytes of device workspace fa_bwd needs: an fp32 dQ accumulator [B,H,N,d], D = rowsum(dO * O)
 * fp32 [B,H,N] (each part 256-byte aligned) and 256 bytes for the main launch's work counter.
 * 0 on invalid sizes. */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/* Backward, bf16 ("48 FlashAttention", block "Tiling и online softmax", paragraph "Backward — тоже
 * без N×N": every probability block is recomputed from Q, K and the saved normaliser instead of
 * being stored; "Flash Attention：如何通过硬件感知优化重塑注意力机制的未来", section 3.2: fp32 gradient
 * accumulation).  Given q, k, v, the forward's o and lse, and the upstream gradient dO
 * (all as produced/consumed by fa_fwd), writes dq, dk, dv (bf16 [B,H,N,d]).
 * workspace: caller-owned device memory of at least fa_bwd_workspace_size() bytes,
 * 256-byte aligned, clobbered; it must not be shared by calls that may overlap.
 * Three kernel launches, in this order: fa_bwd_prep, fa_bwd_main, fa_bwd_dq_convert. */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv,
                 int B, int H, int N, int d, float scale, int causal,
                 const int32_t* key_lens, float dropout_p, uint64_t seed,
                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The three launches of fa_bwd, exposed separately (same arguments, same workspace) so that a
 * caller can time or interleave them.  Calling them in order is equivalent to fa_bwd.
 *  fa_bwd_prep:       D = rowsum(dO * O) into the workspace, clears the dQ accumulator and the
 *                     work counter (fa_bwd_main needs both cleared: run fa_bwd_prep before it).
 *  fa_bwd_main:       dK and dV (written), dQ accumulated (fp32) into the workspace.
 *  fa_bwd_dq_convert: dq = bf16(scale * accumulator). */
FA_API fa_status fa_bwd_prep(const void* o, const void* dO, int B, int H, int N, int d,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);
FA_API fa_status fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dO,
                      void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                      const int32_t* key_lens, float dropout_p, uint64_t seed,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);
FA_API fa_status fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Backward with dQ in a pass of its own: the same arguments and results as fa_bwd (same workspace).
 * Three launches: fa_bwd_prep; the main kernel making dK and dV only; a query-tile-major kernel that
 * recomputes S, P and dP per key block and accumulates dQ = scale * dS K in tensor memory, writing
 * each dQ row once (no fp32 accumulator reductions).  It recomputes two of the five matmuls, so it
 * does more arithmetic than fa_bwd; both are kept so that the two ways of forming dQ that the
 * method allows ("48 FlashAttention", block "Tiling и online softmax": dQ accumulated atomically or
 * in a separate pass) can be compared. */
FA_API fa_status fa_bwd_split(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv,
                       int B, int H, int N, int d, float scale, int causal,
                       const int32_t* key_lens, float dropout_p, uint64_t seed,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Backward that allocates nothing, for callers that cannot allocate device memory: a plugin
 * inside another runtime that owns all device memory and hands it no workspace, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device synchronisation.
 * (The paper has no counterpart: this is an interface convenience of this library.)
 * Same arguments and results as fa_bwd, minus the workspace: the scratch (fp32 dQ accumulator
 * and D, fa_bwd_workspace_size() bytes) lives in a fixed 48 MiB array inside the library, which
 * every GPU that loads the library keeps until the process exits.  Sizes whose scratch exceeds
 * fa_bwd_noalloc_max_scratch() are rejected with FA_ERR_INVALID_ARG.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that device current; make
 * that first call before any stream capture.  All calls share the one array: calls that may
 * overlap on the GPU (other streams, other threads) race and give wrong gradients; serialise
 * them.  Each call clears the part of the array that must start at zero. */
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv,
                         int B, int H, int N, int d, float scale, int causal,
                         const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream);

/* Size in bytes of fa_bwd_noalloc's static scratch array (48 MiB). */
FA_API size_t fa_bwd_noalloc_max_scratch(void);

/* Decode-shaped forward, bf16: Nq new query rows per head (1 <= Nq <= 64) against a cache of Nkv
 * keys ("48 FlashAttention", block "Связи": the attention under vLLM / PagedAttention).
 * q: bf16 [B,H,Nq,d]; k, v: bf16 [B,H,Nkv,d]; writes o (bf16 [B,H,Nq,d]) and lse (fp32 [B,H,Nq]).
 * Sequence b holds L = key_lens[b] valid keys (key_lens: int32 [B] on the device, or NULL for all
 * Nkv); query i is the token at position L - Nq + i, so causal keeps key j <= L - Nq + i and key
 * padding keeps j < L.  A query with no allowed key gets O = 0 and lse = -inf.  No dropout.
 * d in {64, 128}.  The key range of each head is split over CTAs (fa_fwd_decode_split splits
 * per head) that write fp32 partials (m, l, unnormalised O; two per split, one per key half of
 * its 128-key blocks) into the caller's workspace (at least
 * fa_fwd_decode_workspace_size() bytes, 256-byte aligned, clobbered; not shared by calls that may
 * overlap), then a second launch merges them.  Two kernel launches.
 * The workspace size depends on the current device's SM count; with no visible device it is the
 * size for the finest split (512-key chunks), enough on any device.  fa_fwd_decode returns
 * FA_ERR_INVALID_ARG when the workspace is smaller than the current device needs. */
FA_API size_t fa_fwd_decode_workspace_size(int B, int H, int Nq, int Nkv, int d);
/* Number of key-range splits per head that fa_fwd_decode uses for B*H heads of Nkv keys on a device
 * of `sms` SMs (sms <= 0: the finest split).  The split kernel holds one CTA per SM, so the choice
 * minimises waves x (chunk + 256 keys of fixed cost per split) over chunks of whole 128-key blocks,
 * at least 512 keys.  Host arithmetic only; 0 for B, H or Nkv < 1. */
FA_API int fa_fwd_decode_split(int B, int H, int Nkv, int sms);
FA_API fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int Nq, int Nkv, int d, float scale, int causal,
                        const int32_t* key_lens, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/* Heads per group of the backward's head-grouped launch order for sequence length N and head
 * dimension d on a device with l2_bytes of L2: a quarter of L2 divided by the bytes of one head's
 * Q, dO and fp32 dQ accumulator (8 * N * d), rounded to nearest and clamped to [1, 16].  Host-only
 * arithmetic, exposed so that it can be checked without a GPU. */
FA_API int fa_bwd_head_group(int N, int d, size_t l2_bytes);

/* Writes the dropout keep decisions (1 = kept, 0 = dropped) of every element into
 * keep (uint8 [B,H,N,N], device).  For testing the counter hash bit for bit. */
FA_API fa_status fa_dropout_mask(uint8_t* keep, int B, int H, int N, float dropout_p, uint64_t seed,
                          cudaStream_t stream);

/* Test hook: y[i] = 2^x[i] (fp32 device arrays of n elements) by the polynomial exponential that
 * the d = 64 forward runs on the FMA pipe for part of its scores (range reduction x = n + f,
 * a cubic for 2^f with p(0) = 1, n added to the exponent field; x clamped at -127).  Its relative
 * error is below 8.6e-5 for x >= -126; x <= -127 gives exactly 0; x in (-127, -126) gives a value
 * below 2^-126.  For checking that bound. */
FA_API fa_status fa_test_exp2_fma(const float* x, float* y, int n, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears this device's status word.  Returns
 * FA_ERR_TIMEOUT if a bounded wait ran out in any kernel since the last check,
 * FA_ERR_INTERNAL for other device-detected faults, FA_ERR_CUDA if the synchronisation
 * itself failed, FA_OK otherwise. */
FA_API fa_status fa_check(cudaStream_t stream);

/* Description of the last non-OK status returned on the calling thread. */
FA_API const char* fa_get_error(void);

/* Upper bound, in nanoseconds, on every wait inside the kernels (default 2 s; the
 * environment variable FA_WAIT_LIMIT_MS overrides the default).  Applies to later launches. */
FA_API void fa_set_wait_limit_ns(uint64_t ns);

/* Test hook.  Bit 0: the forward's load warp never delivers its first K/V block; bit 1: the
 * backward's load warp never delivers its first Q tile.  Either way the consumers' bounded waits
 * run out, the kernel unwinds and fa_check() returns FA_ERR_TIMEOUT.  0 = normal. */
FA_API void fa_debug_set_flags(int flags);

/* Library version string. */
FA_API const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_FA_H */
