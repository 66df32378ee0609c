/*
 * fa.h - C ABI of a B200 (sm_100a) library of exact, IO-aware fused
 * scaled-dot-product attention: forward and backward.
 *
 * What it computes. For each batch b and head h, with Q, K, V of size N x d
 * ("FlashAttention原理：从原始Attention到FlashAttention", blog.csdn.net/qq_43527718,
 * section 二.2, the standard computation):
 *     S = scale * Q K^T,  P = softmax(S) row by row,  O = P V.
 * The library never forms S or P in global memory: Q is tiled against K/V
 * blocks held on chip and the row softmax is merged block by block with a
 * running maximum and running sum (same page, sections 二.5 and 二.6;
 * "FlashAttention：优化大模型训练的内存与计算效率", cnnetsun.cn, sections 2.1 and
 * 2.2). Only O and the per-row log-sum-exp go back to global memory. The
 * backward recomputes P tile by tile from that stored log-sum-exp instead of
 * reading a stored N x N matrix (blog section 二, "做法", second strategy).
 *
 * Conventions shared by every call:
 *   Layout     q, k, v, o, dO, dq, dk, dv are dense, contiguous [B, H, N, d]
 *              row-major tensors (the [B, H, N, d] shape of the pasted
 *              pseudocode on the blog page, step 1). lse is [B, H, N] fp32.
 *              The grouped-query, variable-length and FP8 calls below state
 *              where theirs differ.
 *   dtypes     q, k, v, dO, dq, dk, dv: bf16. o: bf16 or fp32 in fa_fwd
 *              (o_dtype), bf16 in fa_bwd.
 *   Pointers   device pointers (CUDA global memory of the current device),
 *              each 16-byte aligned. The caller owns every buffer, including
 *              the backward workspace. The library allocates no device memory
 *              at run time. Across calls it keeps, per CUDA context, the
 *              address of fa_bwd_noalloc's fixed scratch array (part of the
 *              loaded module) and which kernels have had their shared-memory
 *              limit raised; per device, the SM count; and, per host thread,
 *              the last CUDA error code.
 *   Sizes      B >= 1, H >= 1, N >= 1 (any value, ragged tails are handled),
 *              d in {64, 128}, B*H*N < 2^31, N <= 2^29 (T <= 2^29 packed).
 *   scale      the factor applied to Q K^T (1/sqrt(d) in the pages' pseudocode,
 *              step 3); any finite value > 0.
 *   causal     0: every key visible. 1: key j visible to query i iff j <= i
 *              (the autoregressive mask named by is_causal in cnnetsun.cn
 *              section 3.1); tiles entirely above the diagonal are skipped
 *              (blog section 二.7, third point).
 *   stream     a cudaStream_t passed as void*; NULL means the legacy default
 *              stream. All work is asynchronous on that stream.
 *   Errors     argument errors come back synchronously, before any launch,
 *              as FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED. A failed launch
 *              returns FA_ERR_CUDA. Every device-side wait in the kernels has
 *              a time limit; if one gives up, the kernel records it in a
 *              device error word and returns early, and fa_get_device_error
 *              reports FA_ERR_TIMEOUT (fa_decode_device_error lists every
 *              bit of that word and its status).
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or scale */
  FA_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (e.g. d = 96) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up */
} fa_status;

typedef enum { FA_BF16 = 0, FA_F32 = 1 } fa_dtype;

/*
 * Forward pass. Writes O (o_dtype) and lse = ln(sum_j exp(scale * q_i . k_j))
 * over visible j, natural log, fp32 (the stored softmax normalisation factor
 * of blog section 二 "做法"; log space per cnnetsun.cn section 2.2).
 * Reads q, k, v once from global memory per CTA's tiles; writes O and lse once.
 * Inputs: q, k, v (bf16 [B,H,N,d]). Outputs: o ([B,H,N,d], o_dtype), lse
 * (fp32 [B,H,N]).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, float scale, int causal, fa_dtype o_dtype,
                 void* stream);

/*
 * Bytes of caller-owned device workspace fa_bwd needs: a fp32 [B,H,N,d]
 * accumulator for dQ, then two fp32 [B,H,N'] per-row arrays (lse in base 2,
 * and the row-dot D = rowsum(dO * O)) with N' = N rounded up to a multiple of
 * 4; each piece rounded up to 256 bytes. Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass. Given the forward inputs, its outputs o (bf16) and lse, and
 * the upstream gradient dO, writes dq, dk, dv (bf16 [B,H,N,d]):
 *     dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO_i * O_i),
 *     dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q,
 * with P recomputed on chip from q, k and lse (blog section 二.5, second point).
 * Launches three kernels, in order on `stream`: the dO.O row-dot kernel
 * (which also zeroes the dQ accumulator), the main kernel (loops over query
 * tiles for each key tile, accumulating dK and dV on chip and adding dQ
 * contributions into the fp32 accumulator), and a kernel that converts the
 * accumulator to bf16 dq.
 * workspace: device pointer, 256-byte aligned, at least
 * fa_bwd_workspace_size(B,H,N,d) bytes (else FA_ERR_INVALID_ARG). Its
 * contents on entry do not matter; on exit they are scratch.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                 int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace. The pages have
 * no counterpart; this exists for callers that may not allocate device
 * memory themselves, such as code inside a host application that owns every
 * GPU allocation, or a latency-critical path where a cudaMalloc is not
 * allowed. It computes exactly what fa_bwd computes, with the same arguments
 * minus the workspace, by the same kernels.
 *
 * Its scratch (the dQ accumulator and two per-row arrays, as sized by
 * fa_bwd_workspace_size) is one fixed device array inside the library of
 * FA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits. Problems with fa_bwd_workspace_size(B,H,N,d) >
 * FA_NOALLOC_SCRATCH_BYTES are rejected with FA_ERR_UNSUPPORTED before any
 * launch. No call allocates: no cudaMalloc, cudaFree or allocating library
 * routine.
 *
 * The first call in each CUDA context (normally one per device: the
 * device's primary context) looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it under the
 * context's unique ID, so a context created later - after cudaDeviceReset,
 * or one the caller makes current through the driver API - looks it up
 * afresh instead of reusing a stale address. Make that first call before any
 * stream capture. Every call shares the one array and
 * the array keeps the last call's contents (the call itself clears what must
 * start at zero), so calls whose work overlaps on the GPU - on different
 * streams, or from different threads - race on it: order them on one stream
 * or synchronise between them.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                         float scale, int causal, void* stream);

/*
 * Grouped-query / multi-query attention (several query heads share one K/V
 * head; "FlashAttention原理：从原始Attention到FlashAttention", blog.csdn.net,
 * related-article notes on MQA/GQA). q, o, dO, dq are [B, H, N, d]; k, v,
 * dk, dv are [B, Hkv, N, d] with H % Hkv == 0, and query head h reads K/V
 * head h / (H / Hkv). Hkv == H is ordinary multi-head attention (what fa_fwd
 * and fa_bwd compute); Hkv == 1 is multi-query attention. dk and dv hold the
 * gradient of each shared K/V head, summed over its group, accumulated on
 * chip over the query heads one CTA covers. lse is [B, H, N]. Every other
 * convention is fa_fwd's and fa_bwd's; Hkv < 1 or H % Hkv != 0 gives
 * FA_ERR_INVALID_ARG.
 *
 * When few K/V heads would leave the GPU short of CTAs, fa_bwd_gqa splits
 * each group's query heads over several CTAs, which add their partial dK and
 * dV into fp32 accumulators in the workspace (zeroed by the row-dot kernel)
 * and two more launches of the convert kernel write dk and dv. Its workspace
 * is fa_bwd_gqa_workspace_size(B, H, Hkv, N, d) bytes: fa_bwd_workspace_size
 * (B, H, N, d) plus, when Hkv < H, two fp32 [B, Hkv, N, d] arrays, each
 * rounded up to 256 bytes (0 for invalid sizes). The split adds fp32 sums in
 * a run-dependent order, so dk and dv may then differ between runs in the
 * last bits.
 */
size_t fa_bwd_gqa_workspace_size(int B, int H, int Hkv, int N, int d);
fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Hkv, int N, int d, float scale, int causal, fa_dtype o_dtype,
                     void* stream);
fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                     int B, int H, int Hkv, int N, int d, float scale, int causal, void* stream);

/*
 * Local-window (band) attention ("Local-Window" among the sparse extensions of
 * "FlashAttention：优化大模型训练的内存与计算效率", cnnetsun.cn, section 6.1):
 * key j is visible to query i iff
 *     i - window_left <= j <= i + window_right,
 * a negative bound meaning no limit on that side. (-1, -1) is full attention,
 * (-1, 0) causal attention, (w, 0) causal attention over the last w + 1
 * keys. The diagonal is always visible, so no row is empty. Only the K/V
 * tiles (forward) or query tiles (backward) that the band touches are
 * visited, so the work is about N * min(N, wl + wr + 1) per head. Grouped
 * K/V heads and every other convention are those of fa_fwd_gqa / fa_bwd_gqa
 * (the backward workspace is fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)
 * bytes). fa_fwd_gqa and fa_bwd_gqa are these calls with (-1, causal ? 0 : -1).
 */
fa_status fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int H, int Hkv, int N, int d, float scale,
                        int window_left, int window_right, fa_dtype o_dtype, void* stream);
fa_status fa_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                        int B, int H, int Hkv, int N, int d, float scale,
                        int window_left, int window_right, void* stream);

/*
 * Variable-length batches (the dynamic-shape support that "FlashAttention：
 * 优化大模型训练的内存与计算效率", cnnetsun.cn, lists among its optimisation
 * directions): B sequences of different lengths packed back to back, with no
 * padding. q, o, dO, dq are [T, H, d] and k, v, dk, dv [T, Hkv, d] bf16,
 * token-major; sequence b owns packed rows [cu_seqlens[b], cu_seqlens[b+1]).
 * lse is fp32 [H, T]. cu_seqlens is a device int32 array of B + 1
 * non-decreasing prefix sums from 0 to at most T (4-byte aligned); every
 * length is at most max_seqlen. Each sequence is attended on its own, with
 * the window (causal: (-1, 0)) applied within the sequence, exactly as if it
 * were a batch of one. The grid covers max_seqlen for every sequence; blocks
 * past the end of a shorter sequence exit at once.
 * Malformed cu_seqlens cannot make a kernel read or write outside the
 * buffers: each entry is clamped to [0, T] and each length to max_seqlen, and
 * fa_get_device_error then reports FA_ERR_INVALID_ARG. The last tile of a
 * sequence reads the packed rows after it and masks them out; a masked
 * product is exactly zero only for finite values, so every row of q, k, v
 * (and of o, lse, dO for the backward) must be finite, as it is when the
 * sequences cover all T rows (cu_seqlens[0] = 0, cu_seqlens[B] = T). The
 * forward leaves the o and lse of rows that no sequence covers untouched; the
 * backward's dq, dk, dv there are unspecified.
 * The backward workspace is fa_bwd_varlen_workspace_size(B, T, H, Hkv, d)
 * bytes (0 for invalid sizes): an fp32 [T, H, d] dQ accumulator, then two
 * fp32 [H][S] statistics arrays with S = T + 4B + 4 rounded up to a multiple
 * of 4 (each sequence's statistics start on a 16-byte boundary), then, when
 * Hkv < H, two fp32 [T, Hkv, d] dK/dV accumulators; each piece rounded up to
 * 256 bytes. Every other convention is fa_fwd_window's/fa_bwd_window's.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens, int B, int max_seqlen, int T, int H, int Hkv, int d,
                        float scale, int window_left, int window_right, fa_dtype o_dtype, void* stream);
size_t fa_bwd_varlen_workspace_size(int B, int T, int H, int Hkv, int d);
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens,
                        void* workspace, size_t ws_bytes, int B, int max_seqlen, int T, int H, int Hkv,
                        int d, float scale, int window_left, int window_right, void* stream);

/*
 * FP8 forward (low-precision inputs, listed among the optimisation directions
 * of "FlashAttention：优化大模型训练的内存与计算效率", cnnetsun.cn). q8 is
 * [B, H, N, 128], k8 and v8 [B, Hkv, N, 128], all 8-bit e4m3 codes (sign,
 * 4-bit exponent with bias 7, 3-bit mantissa; no infinities), each tensor with
 * one fp32 dequantisation scale: the value of a code c of Q is
 * e4m3(c) * q_scale, and likewise for K and V. Computes the attention of the
 * dequantised tensors with the window convention of fa_fwd_window, writing O
 * (bf16 or fp32, [B, H, N, 128]) and lse (fp32 [B, H, N]). Both products run
 * on the tensor cores in e4m3 with fp32 accumulation; the probabilities are
 * rounded to e4m3 (relative error at most 2^-4, absolute at most 2^-10 below
 * 2^-6) before they multiply V, and lse uses the unrounded row sums. d must be
 * 128 (else FA_ERR_UNSUPPORTED); a scale that is not finite and positive gives
 * FA_ERR_INVALID_ARG. There is no FP8 backward.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse,
                     int B, int H, int Hkv, int N, int d, float scale,
                     float q_scale, float k_scale, float v_scale,
                     int window_left, int window_right, fa_dtype o_dtype, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word and
 * returns fa_decode_device_error of it: FA_OK if nothing was recorded since
 * the last call. FA_ERR_CUDA also if the synchronisation or the read failed.
 */
fa_status fa_get_device_error(void* stream);

/*
 * Bits of the device error word that the kernels set (the word is the OR of
 * everything recorded since it was last cleared).
 */
#define FA_DEVERR_TIMEOUT 1u    /* a bounded wait gave up; the kernel returned early */
#define FA_DEVERR_SMEM_ALIGN 2u /* dynamic shared memory was not 1 KB aligned; the kernel did nothing */
#define FA_DEVERR_SEQLENS 4u    /* cu_seqlens entries outside [0, T], decreasing, or longer than max_seqlen */

/*
 * The status a device error word stands for (host only, no CUDA call), in
 * this order of precedence: 0 -> FA_OK; any FA_DEVERR_TIMEOUT ->
 * FA_ERR_TIMEOUT; else FA_DEVERR_SMEM_ALIGN or any bit not listed above ->
 * FA_ERR_CUDA (the launch environment broke a kernel's assumption, no result
 * was computed); else (FA_DEVERR_SEQLENS alone) -> FA_ERR_INVALID_ARG (the
 * kernels clamped the malformed prefix sums; results for those sequences are
 * unspecified).
 */
fa_status fa_decode_device_error(unsigned int word);

/*
 * Measurement hook. After this call, every fa_bwd made by the calling host
 * thread records `before` and `after` (each a cudaEvent_t passed as void*,
 * created by the caller) on its stream immediately before and after the main
 * backward kernel, so that kernel's own duration can be read with
 * cudaEventElapsedTime. Pass NULL, NULL to stop. The events stay owned by the
 * caller and must outlive the fa_bwd calls that record them. Always FA_OK.
 */
fa_status fa_set_bwd_main_events(void* before, void* after);

/*
 * Detail for the most recent FA_ERR_CUDA returned to the calling host thread:
 * the cudaError_t value of the failed runtime call, -1 if a TMA descriptor
 * could not be encoded, 0 if no CUDA failure has been returned.
 */
int fa_last_cuda_error(void);

/*
 * Test hook for the failure-detection path. Launches one thread on `stream`
 * that waits, through the same bounded wait every kernel of this library
 * uses, on a barrier nothing ever completes. After the wait's time limit
 * (about 2 s) it gives up, records the timeout in the device error word and
 * the kernel exits normally, so the next fa_get_device_error(stream) returns
 * FA_ERR_TIMEOUT and the context stays usable. No GPU fault is involved.
 * Returns FA_OK once launched.
 */
fa_status fa_selftest_wait_timeout(void* stream);

/*
 * Test hook for the forward kernel's exp2 on the FMA pipe (Cody-Waite range
 * reduction and a fitted cubic; see fa_fwd.cuh): y[i] = 2^x[i] for n fp32
 * device values, as the softmax computes it for part of its exponentials.
 * Asynchronous on `stream`. FA_ERR_INVALID_ARG for n < 0 or null pointers
 * with n > 0.
 */
fa_status fa_selftest_exp2_fma(const float* x, float* y, long long n, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* fa_strerror(fa_status status);

/* Library version as major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
