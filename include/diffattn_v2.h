/*
 * diffattn_v2.h -- C ABI of the forward Differential Attention V2 operator for NVIDIA B200
 * (sm_100a).
 *
 * What the operator computes. For every batch element b, every query row i and every pair
 * p of adjacent query heads (h1 = 2p, h2 = 2p+1), which share one key/value head
 * g = 2p / (Hq/Hkv) of the grouped-query layout:
 *
 *     A1 = softmax(q[b,i,h1] . K_g^T / sqrt(D))      A2 = softmax(q[b,i,h2] . K_g^T / sqrt(D))
 *     out[b,i,p] = (A1 - lambda[b,i,p] * A2) . V_g
 *
 * over the keys visible from row i (causal: j <= i; decode: j < seqlens[b]).
 * Sources: "Differential Attention (V2)" lesson (AI Engineering from Scratch), section
 * "The differential concept" (equations for A1, A2 and DiffAttn); "Attention variants"
 * lesson, "Build it", Steps 1 and 4 (causal mask, causal diff_attention); "Differential
 * Transformer V2 soll KI-Training stabiler machen", sections "Gemeinsamer KV-Cache statt
 * Spezialkernel" (adjacent heads of one GQA group share K/V) and "Weniger Ausreisser und
 * Gradientenspitzen" (a sigmoid-bounded lambda per token and per head).
 *
 * Conventions shared by every entry point:
 *   - Layout "BSHD": row-major, contiguous, the head dimension D innermost.
 *       prefill  q [B,S,Hq,D]   k, v [B,S,Hkv,D]   lambda fp32 [B,S,Hq/2]   out [B,S,Hq/2,D]
 *       decode   q [B,Hq,D]     kcache, vcache [B,Smax,Hkv,D]   seqlens int32 [B]
 *                lambda fp32 [B,Hq/2]   out [B,Hq/2,D]
 *   - Pairing contract: Hq is even and a multiple of 2*Hkv, so both heads of a pair sit in
 *     the same KV group. Head 2p is the first (+) branch, head 2p+1 the subtracted one.
 *   - Every pointer is a DEVICE pointer (or managed memory) unless stated otherwise. The
 *     caller owns every buffer and the stream; the library never allocates, frees or keeps
 *     a pointer after the call returns.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream) and reentrant:
 *     the library holds no per-call state. A return of DA2_OK means the work was enqueued.
 *     Two pieces of process-wide state exist: the device error word (below), one per device
 *     and shared by every call on every stream of that device, and the no-allocation decode
 *     array of diffattn_v2_decode_noalloc.
 *   - The library caches, per device, the device addresses of its own device variables (the
 *     error word and the no-allocation array), looked up in the context current at the
 *     first call on that device. It supports the device's primary context (what the CUDA
 *     runtime uses by default); the cached addresses do not survive cudaDeviceReset, so a
 *     process that resets a device must not call the library on it afterwards.
 *   - Argument checks happen on the host before anything is launched; a failed check
 *     returns an error and launches nothing. Null pointers, sizes <= 0 (except the B == 0
 *     or S == 0 no-op), an odd Hq, Hq % (2*Hkv) != 0, pointers not 16-byte aligned and a
 *     too-small workspace give DA2_ERR_INVALID. Valid shapes the kernels do not implement
 *     give DA2_ERR_UNSUPPORTED. A failed CUDA call gives DA2_ERR_CUDA.
 *   - Kernels never trap. Every wait inside a kernel is bounded; on expiry the kernel
 *     records an error word on the device and returns; the outputs of that call are then
 *     undefined (a decode whose split gave up never writes that (b, KV head)'s output).
 *     diffattn_v2_device_error() reads and clears the word. There is one word per device,
 *     not per stream: an error raised by a kernel on any stream is reported to (and
 *     cleared by) whichever caller reads the word first.
 *   - The score scale is 1/sqrt(D) for both branches. lambda may be any finite fp32
 *     value (the V2 sigmoid-bounded value in (0,1), or a V1 value that may be negative or
 *     above 1).
 */
#ifndef DIFFATTN_V2_H_
#define DIFFATTN_V2_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define DA2_API __attribute__((visibility("default")))
#else
#define DA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle; identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* da2_stream_t;

/* Status codes returned by every entry point. */
enum {
  DA2_OK = 0,
  DA2_ERR_INVALID = -1,     /* an argument failed a host-side check; nothing launched   */
  DA2_ERR_UNSUPPORTED = -2, /* valid arguments this build does not implement            */
  DA2_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch, attribute, symbol)   */
  DA2_ERR_DEVICE = -4       /* a kernel recorded an internal error (bounded wait expired) */
};

/* Library version: 100 * major + minor. */
DA2_API int diffattn_v2_version(void);

/* Human-readable name of a status code (static string, never NULL). */
DA2_API const char* diffattn_v2_status_string(int status);

/*
 * Causal (or full) prefill, bf16 in / bf16 out, fp32 accumulation and softmax.
 * Source: "The differential concept" (DiffAttn = (A1 - lambda A2) V) with the causal
 * mask of the attention-variants lesson, Step 1, and the V2 head pairing above.
 *   q      bf16 [B,S,Hq,D]        k, v  bf16 [B,S,Hkv,D]
 *   lambda fp32 [B,S,Hq/2]        out   bf16 [B,S,Hq/2,D] (fully overwritten)
 *   causal 1: key j visible from query i iff j <= i (Sq == Sk == S); 0: all S keys visible.
 * Supported: D == 128. Other D give DA2_ERR_UNSUPPORTED. Each (b, p) output row is
 * O1/l1 - lambda*O2/l2 formed in fp32 and rounded once to bf16 (round to nearest even).
 * Kernel: tcgen05 tensor-core MMAs with TMEM accumulators, TMA-staged K/V tiles loaded
 * once per pair, two online softmaxes. B == 0 or S == 0 is a no-op returning DA2_OK.
 */
DA2_API int diffattn_v2_prefill(const void* q, const void* k, const void* v, const float* lambda,
                        void* out, int B, int S, int Hq, int Hkv, int D, int causal,
                        da2_stream_t stream);

/*
 * Causal prefill with a sliding window, bf16 in / bf16 out: query i sees keys
 * max(0, i - window + 1) .. i (the window holds the query's own key). This is DiffAttn in a
 * sliding-window layer, the hybrid the "Differential Attention (V2)" lesson's "Use it"
 * section names, with the window mask of the "Attention variants" lesson, "Build it",
 * Step 2. Arguments, layout and semantics as diffattn_v2_prefill with causal = 1;
 * window >= 1 (window >= S is the plain causal prefill); window < 1 gives DA2_ERR_INVALID.
 * Only the KV tiles that intersect a query tile's windows are read.
 */
DA2_API int diffattn_v2_prefill_window(const void* q, const void* k, const void* v, const float* lambda,
                                       void* out, int B, int S, int Hq, int Hkv, int D, int window,
                                       da2_stream_t stream);

/*
 * Prefill of B sequences of different lengths packed along the token axis (the layout of
 * serving engines), bf16 in / bf16 out. Sequence b is tokens cu_seqlens[b] ..
 * cu_seqlens[b+1]-1; each sequence is an independent prefill (its queries see only its own
 * keys, causally when causal = 1).
 *   q bf16 [T,Hq,D]   k, v bf16 [T,Hkv,D]   lambda fp32 [T,Hq/2]   out bf16 [T,Hq/2,D]
 *   cu_seqlens int32 [B+1] (device), non-decreasing, cu_seqlens[0] = 0, cu_seqlens[B] = T
 *   max_seqlen >= the longest sequence (bounds the row tiles a sequence can have; rows of a
 *   sequence past max_seqlen are not computed)
 *   total_tokens = T
 * The caller guarantees the cu_seqlens contract; the kernel reads it on the device, so the
 * call needs no host synchronisation. Supported: D == 128. Zero-length sequences are allowed.
 * Schedule: up to 256 sequences, persistent CTAs (one per SM) sort the sequences by length
 * on the device and deal out only the non-empty (sequence, pair, 128-row tile) items; with
 * more sequences every item of the B x pairs x ceil(max_seqlen/128) grid gets its own CTA.
 */
DA2_API int diffattn_v2_prefill_varlen(const void* q, const void* k, const void* v, const float* lambda,
                                       void* out, const int32_t* cu_seqlens, int B, int max_seqlen,
                                       int total_tokens, int Hq, int Hkv, int D, int causal,
                                       da2_stream_t stream);

/*
 * The same operator in fp32 end to end (CUDA-core arithmetic, no tensor cores), for
 * callers that need results within ~1e-5 of exact. q, k, v, out are fp32 with the prefill
 * layout above. Supported: D in {64, 128}. Same argument checks and semantics.
 */
DA2_API int diffattn_v2_prefill_f32(const float* q, const float* k, const float* v,
                            const float* lambda, float* out, int B, int S, int Hq, int Hkv,
                            int D, int causal, da2_stream_t stream);

/*
 * Training forward: diffattn_v2_prefill (same arguments, checks and out) that also writes
 * what the backward pass needs ("Differential Transformer V2 soll KI-Training stabiler
 * machen": V2 is meant for pretraining, so the operator carries gradients):
 *   o_branch bf16 [B,S,Hq,D]  O_b = softmax(Q_b K^T / sqrt(D)) V of every query head, each
 *                             normalised on its own (head 2p is branch 1 of pair p, 2p+1
 *                             branch 2), so out = O_{2p} - lambda * O_{2p+1} up to rounding
 *   lse      fp32 [B,S,Hq]    log2-domain log-sum-exp of the head's scaled scores:
 *                             softmax row = 2^(s * log2(e) / sqrt(D) - lse)
 * Caller-owned device buffers, 16-byte aligned; D == 128.
 */
DA2_API int diffattn_v2_prefill_train(const void* q, const void* k, const void* v, const float* lambda,
                                      void* out, void* o_branch, float* lse, int B, int S, int Hq,
                                      int Hkv, int D, int causal, da2_stream_t stream);

/* Scratch (bytes) diffattn_v2_backward needs: fp32 [B,S,Hq] row terms; 0 for invalid sizes. */
DA2_API size_t diffattn_v2_backward_workspace_size(int B, int S, int Hq);

/*
 * Gradients of the bf16 prefill given dout = dL/d(out), bf16 [B,S,Hq/2,D]. Chain rule of
 * out = softmax(Q_1 K^T/sqrt(D)) V - lambda * softmax(Q_2 K^T/sqrt(D)) V ("Differential
 * Attention (V2)" lesson, "The differential concept"; causal mask of the "Attention
 * variants" lesson):
 *   dq bf16 [B,S,Hq,D]    dL/dQ of every query head (both branches of every pair)
 *   dk, dv bf16 [B,S,Hkv,D]  summed over the query heads of each KV head's group
 *   dlambda fp32 [B,S,Hq/2]  dL/dlambda = -dout . O_2 per token and pair
 * Inputs: q, k, v, lambda as given to diffattn_v2_prefill_train, and the o_branch and lse it
 * wrote. workspace: at least diffattn_v2_backward_workspace_size(B, S, Hq) bytes of device
 * memory, no state between calls. Every output is overwritten (nothing accumulates into
 * it); the result is deterministic (no atomics). Supported: D == 128, causal 0 or 1.
 * Errors: DA2_ERR_INVALID for bad sizes, null or unaligned pointers, short workspace;
 * DA2_ERR_UNSUPPORTED for other D or grids past the launch limits (B or Hq > 65535).
 */
DA2_API int diffattn_v2_backward(const void* q, const void* k, const void* v, const float* lambda,
                                 const void* o_branch, const float* lse, const void* dout, void* dq,
                                 void* dk, void* dv, float* dlambda, int B, int S, int Hq, int Hkv, int D,
                                 int causal, void* workspace, size_t workspace_bytes,
                                 da2_stream_t stream);

/*
 * Training forward and backward of the causal sliding-window prefill (hybrid layers; query
 * i sees keys i-window+1 .. i, "Attention variants" lesson, Step 2): the arguments, layouts,
 * workspace (diffattn_v2_backward_workspace_size) and semantics of diffattn_v2_prefill_train
 * and diffattn_v2_backward with `window` (>= 1; window >= S is the plain causal pass) in place
 * of `causal`. Only the KV tiles inside the windows are read.
 */
DA2_API int diffattn_v2_prefill_window_train(const void* q, const void* k, const void* v, const float* lambda,
                                             void* out, void* o_branch, float* lse, int B, int S, int Hq,
                                             int Hkv, int D, int window, da2_stream_t stream);
DA2_API int diffattn_v2_backward_window(const void* q, const void* k, const void* v, const float* lambda,
                                        const void* o_branch, const float* lse, const void* dout, void* dq,
                                        void* dk, void* dv, float* dlambda, int B, int S, int Hq, int Hkv,
                                        int D, int window, void* workspace, size_t workspace_bytes,
                                        da2_stream_t stream);

/*
 * Training forward and backward for B sequences packed along the token axis (the layout of
 * diffattn_v2_prefill_varlen; pretraining on packed documents). Every sequence is an
 * independent prefill, so its gradients are those of its own prefill:
 *   q bf16 [T,Hq,D]  k, v bf16 [T,Hkv,D]  lambda fp32 [T,Hq/2]  out, dout bf16 [T,Hq/2,D]
 *   o_branch bf16 [T,Hq,D]  lse fp32 [T,Hq]   (written by the training forward, read back)
 *   dq bf16 [T,Hq,D]  dk, dv bf16 [T,Hkv,D]  dlambda fp32 [T,Hq/2]   (overwritten)
 *   cu_seqlens int32 [B+1] (device): sequence b is tokens cu_seqlens[b] .. cu_seqlens[b+1]-1;
 *   max_seqlen >= the longest sequence; total_tokens = T.
 * The backward's workspace: diffattn_v2_backward_varlen_workspace_size(B, T, Hq) bytes of
 * device memory (the row terms of every sequence padded to 128 rows, and B+1 offsets);
 * sizes depend on host-known B and T only, so no host synchronisation is needed. Same
 * checks, semantics and determinism as the [B,S] calls; D == 128.
 */
DA2_API int diffattn_v2_prefill_varlen_train(const void* q, const void* k, const void* v, const float* lambda,
                                             void* out, void* o_branch, float* lse, const int32_t* cu_seqlens,
                                             int B, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                                             int causal, da2_stream_t stream);
DA2_API size_t diffattn_v2_backward_varlen_workspace_size(int B, int total_tokens, int Hq);
DA2_API int diffattn_v2_backward_varlen(const void* q, const void* k, const void* v, const float* lambda,
                                        const void* o_branch, const float* lse, const void* dout, void* dq,
                                        void* dk, void* dv, float* dlambda, const int32_t* cu_seqlens, int B,
                                        int max_seqlen, int total_tokens, int Hq, int Hkv, int D, int causal,
                                        void* workspace, size_t workspace_bytes, da2_stream_t stream);

/*
 * The same training pair with the causal sliding window inside every packed sequence (the
 * mask of diffattn_v2_prefill_varlen_window: query i of a sequence sees that sequence's keys
 * max(0, i-window+1) .. i). Layouts, workspace (diffattn_v2_backward_varlen_workspace_size)
 * and checks as above; window >= 1 (else DA2_ERR_INVALID), window >= max_seqlen is the plain
 * causal pair. Sources: the "Attention variants" lesson's sliding-window step with the packed
 * layout above.
 */
DA2_API int diffattn_v2_prefill_varlen_window_train(const void* q, const void* k, const void* v,
                                                    const float* lambda, void* out, void* o_branch, float* lse,
                                                    const int32_t* cu_seqlens, int B, int max_seqlen,
                                                    int total_tokens, int Hq, int Hkv, int D, int window,
                                                    da2_stream_t stream);
DA2_API int diffattn_v2_backward_varlen_window(const void* q, const void* k, const void* v, const float* lambda,
                                               const void* o_branch, const float* lse, const void* dout, void* dq,
                                               void* dk, void* dv, float* dlambda, const int32_t* cu_seqlens,
                                               int B, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                                               int window, void* workspace, size_t workspace_bytes,
                                               da2_stream_t stream);

/*
 * Workspace (bytes) that diffattn_v2_decode needs for these sizes: the per-split partial
 * results (running max, running sum and unnormalised output of each head), fp32. Returns 0
 * for invalid sizes. The workspace holds no state between calls.
 */
DA2_API size_t diffattn_v2_decode_workspace_size(int B, int Smax, int Hq, int Hkv, int D);

/*
 * One decode step, bf16 in / bf16 out: the new token of each sequence attends to its
 * cached keys [0, seqlens[b]) (the new key and value are already appended by the caller).
 * Source: "Differential Attention (V2)" lesson, "V1 vs V2" (the KV cache is read once per
 * step for both branches; arithmetic intensity doubles) and the DiffAttn equation.
 *   q        bf16 [B,Hq,D]            kcache, vcache bf16 [B,Smax,Hkv,D]
 *   seqlens  int32 [B] (device), each clamped on the device to [0, Smax]
 *   lambda   fp32 [B,Hq/2]            out bf16 [B,Hq/2,D] (fully overwritten)
 *   workspace device buffer of at least diffattn_v2_decode_workspace_size() bytes,
 *            16-byte aligned, owned by the caller; calls that share one workspace must not
 *            overlap on the GPU.
 * A sequence with seqlens[b] == 0 gets an all-zero output. Supported: D == 128 and a GQA
 * group size Hq/Hkv in {2, 4, 8, 16}. One kernel after a small memset of the workspace's
 * split counters: split-KV streaming CTAs (TMA-staged K/V, every visible K/V row read once
 * for all query heads of the group), the last of a (b, KV head)'s splits merging the
 * per-split (max, sum, output) partials of both branches. The workspace needs no
 * initialisation. The grid is sized from Smax on the host, so the call needs no host
 * synchronisation.
 */
DA2_API int diffattn_v2_decode(const void* q, const void* kcache, const void* vcache,
                       const int32_t* seqlens, const float* lambda, void* out, int B, int Smax,
                       int Hq, int Hkv, int D, void* workspace, size_t workspace_bytes,
                       da2_stream_t stream);

/*
 * bf16 decode step of a sliding-window layer: as diffattn_v2_decode, but sequence b's new
 * token sees only its last `window` keys, [max(0, seqlens[b]-window), seqlens[b]) (the mask of
 * the "Attention variants" lesson's sliding-window step, for the hybrid layers of the
 * "Differential Attention (V2)" lesson's "Use it" section). The splits start at the 64-token
 * boundary below the window, so keys before it are not read, and are planned over the
 * window's span when that needs no more of them than the plain decode. Same layouts, workspace size
 * (diffattn_v2_decode_workspace_size) and checks as diffattn_v2_decode, plus
 * DA2_ERR_INVALID for window < 1; window >= Smax is the plain decode.
 */
DA2_API int diffattn_v2_decode_window(const void* q, const void* kcache, const void* vcache,
                                      const int32_t* seqlens, const float* lambda, void* out, int B, int Smax,
                                      int Hq, int Hkv, int D, int window, void* workspace,
                                      size_t workspace_bytes, da2_stream_t stream);

/*
 * The sliding-window decode step over a paged cache: diffattn_v2_decode_paged's layouts with
 * diffattn_v2_decode_window's mask. Block-table entries of pages that hold only keys before
 * a sequence's window are not read (a serving engine may already have released them).
 * Checks as diffattn_v2_decode_paged, plus DA2_ERR_INVALID for window < 1.
 */
DA2_API int diffattn_v2_decode_paged_window(const void* q, const void* kpages, const void* vpages,
                                            const int32_t* block_table, const int32_t* seqlens,
                                            const float* lambda, void* out, int B, int max_pages, int page_size,
                                            int num_pages, int Hq, int Hkv, int D, int window, void* workspace,
                                            size_t workspace_bytes, da2_stream_t stream);

/*
 * The bf16 decode step over a paged KV cache (the layout serving engines keep): the caches
 * are pages of page_size tokens, and logical token t of sequence b is row t % page_size of
 * page block_table[b * max_pages + t / page_size].
 *   kpages, vpages bf16 [num_pages, page_size, Hkv, D]    block_table int32 [B, max_pages]
 *   q, seqlens, lambda, out as in diffattn_v2_decode; seqlens[b] is clamped to
 *   [0, max_pages * page_size]
 *   workspace: diffattn_v2_decode_workspace_size(B, max_pages * page_size, Hq, Hkv, D) bytes
 * page_size is a power of two in [8, 4096]. Entries of block_table past a sequence's last
 * page are never read. Same kernels, arithmetic and results as diffattn_v2_decode on the
 * gathered cache with Smax = max_pages * page_size (bit for bit). Source: the lesson's "Use
 * it" section (integration into the vLLM and SGLang serving engines) and "V1 vs V2" (the
 * cache is read once per step).
 */
DA2_API int diffattn_v2_decode_paged(const void* q, const void* kpages, const void* vpages,
                                     const int32_t* block_table, const int32_t* seqlens,
                                     const float* lambda, void* out, int B, int max_pages, int page_size,
                                     int num_pages, int Hq, int Hkv, int D, void* workspace,
                                     size_t workspace_bytes, da2_stream_t stream);

/*
 * Decode of T new tokens per sequence in one step (e.g. verifying T speculative tokens),
 * bf16 in / bf16 out. The caches already hold all T new keys; new token t of sequence b
 * attends to keys [0, seqlens[b] - T + t + 1), i.e. causally among the new tokens. Source:
 * the lesson's compatibility table (speculative decoding works with DIFF V2: the attention
 * change is invisible to the decoding loop) and the DiffAttn equation.
 *   q bf16 [B,T,Hq,D]   lambda fp32 [B,T,Hq/2]   out bf16 [B,T,Hq/2,D]
 *   caches, seqlens as in diffattn_v2_decode (seqlens[b] >= T; a token without visible keys
 *   gets a zero output)
 *   workspace: diffattn_v2_decode_multi_workspace_size(B, T, Smax, Hq, Hkv, D) bytes
 * The (token, head) pairs of a GQA group share one pass over the cache. Supported: D == 128,
 * group size Hq/Hkv in {2, 4, 8, 16} with T * group <= 16. T == 1 equals diffattn_v2_decode.
 */
DA2_API size_t diffattn_v2_decode_multi_workspace_size(int B, int T, int Smax, int Hq, int Hkv, int D);
DA2_API int diffattn_v2_decode_multi(const void* q, const void* kcache, const void* vcache,
                                     const int32_t* seqlens, const float* lambda, void* out, int B, int T,
                                     int Smax, int Hq, int Hkv, int D, void* workspace, size_t workspace_bytes,
                                     da2_stream_t stream);

/*
 * The decode step in fp32 end to end (CUDA cores), same layout with fp32 q, caches and
 * out, no workspace. Supported: D in {64, 128}.
 */
DA2_API int diffattn_v2_decode_f32(const float* q, const float* kcache, const float* vcache,
                           const int32_t* seqlens, const float* lambda, float* out, int B,
                           int Smax, int Hq, int Hkv, int D, da2_stream_t stream);

/*
 * V1-style lambda: lambda_p = exp(lq1_p . lk1_p) - exp(lq2_p . lk2_p) + lambda_init, one
 * value per pair, written to `rows` consecutive rows of n_pairs values each
 * (lambda_out[r*n_pairs + p], fp32), so the result can feed the decode ([B,Hq/2], rows=B)
 * or prefill ([B,S,Hq/2], rows=B*S) lambda argument directly.
 * Source: "Differential Attention (V2)" lesson, "The differential concept" (the lambda
 * re-parameterisation; lambda_init a small positive number such as 0.8; the value can be
 * negative).
 *   lq1, lk1, lq2, lk2  fp32 [n_pairs, d] (device)     lambda_out fp32 [rows, n_pairs]
 * Computed in fp32 with the accurate expf. Requires n_pairs > 0, d > 0, rows >= 0.
 */
DA2_API int diffattn_v2_lambda_v1(const float* lq1, const float* lk1, const float* lq2,
                          const float* lk2, float lambda_init, int n_pairs, int d, int rows,
                          float* lambda_out, da2_stream_t stream);

/*
 * The bf16 decode step of diffattn_v2_decode (same arguments, layout, semantics and kernels)
 * without a workspace argument, for callers that cannot allocate device memory: serving
 * engines that give nearly all HBM to a KV-cache pool or caching allocator up front, plugin
 * interfaces that hand over only input and output buffers, and loops that must not take
 * the device-wide synchronisation an allocation may imply. The pages describe no such entry
 * point; it has no counterpart there.
 *   - The per-split partials live in a fixed 16 MiB device array inside the library
 *     (16777216 bytes). Every GPU that loads the library holds that array until the process
 *     exits. The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine.
 *   - Sizes whose partials need more than the array, i.e. whenever
 *     diffattn_v2_decode_workspace_size(B, Smax, Hq, Hkv, D) > 16777216, are refused with
 *     DA2_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on a device (with that device current) looks up the array's device
 *     address once (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the one array, and it keeps the last call's contents
 *     (nothing in it needs to start at zero). Calls that overlap on the GPU -- on different
 *     streams, or from different host threads without ordering -- race on it and give wrong
 *     results: serialise them.
 */
DA2_API int diffattn_v2_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                       const int32_t* seqlens, const float* lambda, void* out, int B,
                                       int Smax, int Hq, int Hkv, int D, da2_stream_t stream);

/*
 * V2 lambda: lambda[t, p] = sigmoid(x[t] . w_lambda[:, p] + bias[p]), one value per token and
 * per pair, bounded to (0, 1). Source: "Differential Transformer V2 soll KI-Training stabiler
 * machen", section "Weniger Ausreisser und Gradientenspitzen" (V2 projects a sigmoid-bounded
 * lambda for every token and head instead of V1's per-head normalisation). The projection
 * input is the token's hidden state; whether it has a bias is not fixed by the pages, so
 * bias may be NULL.
 *   x        bf16 [T, d_model]         w_lambda bf16 [d_model, n_pairs]
 *   bias     fp32 [n_pairs] or NULL    lambda_out fp32 [T, n_pairs] (the prefill/decode
 *                                      lambda layout when T = B*S or T = B)
 * bf16 products accumulated in fp32 on the 5th-generation tensor cores (tcgen05, one CTA per
 * 128 tokens); sigmoid with the accurate expf.
 * Supported: d_model % 64 == 0, n_pairs % 8 == 0 and n_pairs <= 64 (else DA2_ERR_UNSUPPORTED).
 */
DA2_API int diffattn_v2_lambda_v2(const void* x, const void* w_lambda, const float* bias, int T, int d_model,
                                  int n_pairs, float* lambda_out, da2_stream_t stream);

/*
 * Causal sliding-window prefill of packed sequences: diffattn_v2_prefill_varlen's layouts and
 * sequence rules with diffattn_v2_prefill_window's mask inside every sequence (query i of a
 * sequence sees that sequence's keys max(0, i-window+1) .. i). Sources: the "Attention
 * variants" lesson, sliding-window step, and the hybrid layers of the "Differential Attention
 * (V2)" lesson's "Use it" section, with the packed layout serving engines use. window >= 1;
 * window >= max_seqlen is the plain causal packed prefill. Host checks and errors as
 * diffattn_v2_prefill_varlen, plus DA2_ERR_INVALID for window < 1.
 */
DA2_API int diffattn_v2_prefill_varlen_window(const void* q, const void* k, const void* v, const float* lambda,
                                              void* out, const int32_t* cu_seqlens, int B, int max_seqlen,
                                              int total_tokens, int Hq, int Hkv, int D, int window,
                                              da2_stream_t stream);

/*
 * bf16 prefill with the V2 lambda fused into the kernel: the same output as
 * diffattn_v2_prefill with lambda[b,s,p] = sigmoid(x[b,s] . w_lambda_t[p] + bias[p]) (the
 * projection of diffattn_v2_lambda_v2), computed per work item by two otherwise idle warps of
 * the prefill kernel instead of by a separate launch. Sources: "Differential Transformer V2
 * soll KI-Training stabiler machen", section "Weniger Ausreisser und Gradientenspitzen" (the
 * lambda), and the prefill's sources above.
 *   q, k, v, out      as diffattn_v2_prefill ([B,S] layouts, D == 128)
 *   x                 bf16 [B, S, d_model] token hidden states
 *   w_lambda_t        bf16 [Hq/2, d_model]: the projection TRANSPOSED, one row per pair
 *                     (w_lambda_t[p][j] = w_lambda[j][p] of diffattn_v2_lambda_v2)
 *   bias              fp32 [Hq/2] or NULL
 *   lambda_out        fp32 [B, S, Hq/2] or NULL: a copy of the computed lambda (the layout a
 *                     training backward reads)
 * Every pair's work items read their rows of x again (Hq/2 times in all), so this form costs
 * more memory traffic than diffattn_v2_lambda_v2 followed by diffattn_v2_prefill; it exists
 * for callers that want one launch. Host checks and errors as diffattn_v2_prefill, plus:
 * d_model > 0 and a multiple of 8, x and w_lambda_t non-NULL and 16-byte aligned, bias and
 * lambda_out NULL or 16-byte aligned.
 */
DA2_API int diffattn_v2_prefill_fused_lambda(const void* q, const void* k, const void* v, const void* x,
                                             const void* w_lambda_t, const float* bias, void* out,
                                             float* lambda_out, int B, int S, int Hq, int Hkv, int D, int d_model,
                                             int causal, da2_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the device error word that kernels set when a
 * bounded wait expires. *code receives 0 when no kernel reported an error, else the code
 * of the first error recorded (a pipeline wait expired: 1 = in a prefill, 2 = in a decode,
 * 3 = in a backward kernel, 5 = in the V2 lambda projection; 4 = an index outside its extent, reported only by the
 * bounds-checking build libdiffattn_v2_debug.so, whose kernels check their shared-memory,
 * tensor-memory and global indices and skip an access that would leave its extent). The word belongs to the current device, not to `stream`: it
 * holds the first error of a kernel on ANY stream of the device since it was last cleared,
 * and reading it clears it for every caller. Synchronising `stream` only orders the read
 * after this stream's kernels; kernels of other streams still running may set it later.
 * Returns DA2_ERR_DEVICE when *code != 0, DA2_OK when it is 0, DA2_ERR_CUDA on a CUDA
 * failure. `code` is a HOST pointer and may be NULL.
 */
DA2_API int diffattn_v2_device_error(int* code, da2_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* DIFFATTN_V2_H_ */
