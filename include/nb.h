/*
 * nb.h - C ABI of the B200 (sm_100a) banded block-sparse local attention and
 * the fused 2-bit DNA k-mer tokenizer.
 *
 * The operations follow the NucleoByte page ("NucleoByte: GPU-Accelerated
 * Block-Sparse Genomic Language Model"):
 *   - section 3 "Mathematical Foundations", subsection "Localized Block-Sparse
 *     Attention Matrix": blocks of B = 32 tokens; query block i attends key
 *     block j only when |i - j| <= R;
 *   - section 3, "Softmax Normalization & Online Numerical Stability":
 *     S = Q K^T / sqrt(d), online softmax with running max and running sum;
 *   - section 3, "Custom Backpropagation": row term D_i = sum_k dO_ik O_ik and
 *     dS_ij = P_ij (dO_i V_j^T - D_i);
 *   - sections 1-2 ("Padding Waste", "Dynamic Ceiling Hardware Alignment"):
 *     sequences padded to a multiple of 32, keys past the true length masked;
 *   - sections 1, 2 and 5 ("Token Blur", "Fused 2-Bit Tokenization",
 *     "Architecture Size"): 2-bit bases, sliding-window 6-mer IDs.
 *
 * Conventions shared by every call:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise (only
 *     nb_attn_fwd_bwd_host and nb_batch_ceiling take host tensors).  The
 *     caller owns every buffer; no call allocates device memory.  The library
 *     keeps no state between calls except per-device caches (device
 *     properties, the device addresses of its two __device__ variables) and
 *     those variables: the kernel error word read by nb_kernel_error (4 bytes)
 *     and the fixed scratch array of nb_attn_bwd_noalloc
 *     (NB_NOALLOC_SCRATCH_BYTES = 64 MiB), which loading the library's device
 *     code reserves on every GPU it runs on, until the process exits.  The
 *     address caches assume the device's primary context lives as long as
 *     the process: resetting a device (cudaDeviceReset) after a call of this
 *     library on it is not supported.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Arguments are validated on the host first: an invalid
 *     call returns a negative nb_status and launches nothing.  A failed launch
 *     returns NB_ERR_CUDA.  Kernels never trap.
 *   - Attention tensors are [batch, heads, n, d] contiguous with d innermost;
 *     log-sum-exp and the row term are [batch, heads, n] fp32.  n must be a
 *     multiple of 32 and d is 64 or 128.  Tensor pointers must be 16-byte
 *     aligned.
 *   - `lengths` (optional, int32 [batch], device) gives each sequence's true
 *     length L_b in [0, n]; NULL means every L_b = n.  Keys k >= L_b are
 *     masked.  Rows q >= L_b are padding: O, dQ, dK, dV are written as 0 there
 *     and log-sum-exp as -inf.  Values outside [0, n] are clamped into it on
 *     the device (they cannot be checked on the host).
 *   - The softmax scale is fixed at 1/sqrt(d).
 */
#ifndef NB_H_
#define NB_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NB_API __attribute__((visibility("default")))
#else
#define NB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nb_status {
  NB_OK = 0,
  NB_ERR_INVALID_ARG = -1, /* null pointer, bad size, n % 32 != 0, R < 0, ... */
  NB_ERR_UNSUPPORTED = -2, /* valid request this build does not implement (d, dtype, k) */
  NB_ERR_MISALIGNED = -3,  /* a tensor pointer is not 16-byte aligned */
  NB_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  NB_ERR_WORKSPACE = -5,   /* workspace pointer null/misaligned or too small */
  NB_ERR_DEVICE = -6       /* the current device is not an sm_100 (B200-class) GPU */
} nb_status;

typedef enum nb_dtype {
  NB_F32 = 0,  /* fp32 storage, fp32 arithmetic (CUDA cores) */
  NB_BF16 = 1  /* bf16 storage, fp32 accumulation (tensor cores) */
} nb_dtype;

#define NB_BLOCK 32 /* the block size B of the band */

/* Human-readable name of a status code.  Never returns NULL. */
NB_API const char* nb_status_string(int status);

/* ABI version of this library (major * 100 + minor). */
NB_API int nb_abi_version(void);

/*
 * nb_kernel_error - report whether a kernel gave up waiting.  Every wait inside
 * the tensor-core kernels is bounded (2 s); a kernel that runs out records a
 * non-zero site code in a device word, frees its tensor memory and returns, so
 * the context stays usable (its outputs are then undefined).  This call
 * synchronises the current device, stores the recorded code (0 = none) in
 * *code and, when `clear` is non-zero, resets it.
 */
NB_API nb_status nb_kernel_error(int* code, int clear);

/*
 * nb_attn_fwd - banded block-sparse local attention, forward.
 *   O[b,h,q,:] = sum_k P[q,k] V[b,h,k,:], P = softmax over the visible keys of
 *   S = Q K^T / sqrt(d); visible: |q/32 - k/32| <= R and k < L_b.
 *   (NucleoByte page, section 3: band predicate, scores, online softmax.)
 * q, k, v  in : [batch, heads, n, d] of `dtype`.
 * o        out: [batch, heads, n, d] of `dtype`.
 * lse      out: [batch, heads, n] fp32, natural-log log-sum-exp of each row's
 *               visible scaled scores (the input the backward needs); may be
 *               NULL when not wanted.
 * lengths  in : int32 [batch] or NULL (see conventions).
 * batch, heads >= 0; n >= 0 and a multiple of 32; d in {64, 128}; R >= 0.
 * dtype: NB_F32 or NB_BF16.  stream: cudaStream_t.
 * Empty problems (batch*heads*n == 0) return NB_OK without a launch.
 */
NB_API nb_status nb_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int32_t* lengths, int batch, int heads, int n, int d, int R,
                      int dtype, void* stream);

/*
 * nb_attn_bwd_workspace_size - bytes of device workspace nb_attn_bwd needs
 * for this shape (0 for an empty problem).  Returns 0 for invalid arguments.
 */
NB_API size_t nb_attn_bwd_workspace_size(int batch, int heads, int n, int d, int dtype);

/*
 * nb_attn_bwd - backward of nb_attn_fwd, recomputing P from the stored
 * log-sum-exp.  (NucleoByte page, section 3 "Custom Backpropagation":
 * D_i = sum_k dO_ik O_ik, dS = P (dO V^T - D); dV = P^T dO, dQ = dS K / sqrt(d),
 * dK = dS^T Q / sqrt(d).)
 * q, k, v   in : the forward's inputs.
 * o, lse    in : the forward's outputs for the same inputs (lse required).
 * dout      in : dL/dO, [batch, heads, n, d] of `dtype`; rows >= L_b ignored.
 * dq, dk, dv out: [batch, heads, n, d] of `dtype`; must not alias the inputs.
 * workspace     : device scratch of at least nb_attn_bwd_workspace_size(...)
 *                 bytes, 256-byte aligned, owned by the caller; its contents on
 *                 entry do not matter and are clobbered.  It must not be used
 *                 by another call that runs concurrently on the GPU.
 * dK and dV are deterministic; dQ is accumulated with fp32 atomics and may
 * differ in the last bits between runs.
 * Currently NB_BF16 only (NB_F32 returns NB_ERR_UNSUPPORTED).
 */
NB_API nb_status nb_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, const int32_t* lengths, void* dq,
                      void* dk, void* dv, void* workspace, size_t workspace_bytes, int batch,
                      int heads, int n, int d, int R, int dtype, void* stream);

/*
 * nb_attn_fwd_causal / nb_attn_bwd_causal - the causal band.  The NucleoByte
 * page's band is symmetric; this is its causal restriction (the plainest
 * reading of a causal band, a variant the page does not print): query q in
 * block i attends key k in block j only when i - R <= j <= i and k <= q (and
 * k < L_b).  Same arguments, layouts, workspace and errors as nb_attn_fwd /
 * nb_attn_bwd; the fp32 forward is supported, the backward is bf16 only.
 */
NB_API nb_status nb_attn_fwd_causal(const void* q, const void* k, const void* v, void* o,
                                    float* lse, const int32_t* lengths, int batch, int heads,
                                    int n, int d, int R, int dtype, void* stream);
NB_API nb_status nb_attn_bwd_causal(const void* q, const void* k, const void* v, const void* o,
                                    const void* dout, const float* lse, const int32_t* lengths,
                                    void* dq, void* dk, void* dv, void* workspace,
                                    size_t workspace_bytes, int batch, int heads, int n, int d,
                                    int R, int dtype, void* stream);

/*
 * nb_attn_fwd_bwd_host - forward then backward (nb_attn_fwd, nb_attn_bwd, or
 * their causal forms when `causal` is non-zero) of tensors that live in HOST
 * memory: the training step of one attention layer for a caller whose
 * activations are on the host.  (NucleoByte page, section 3: the forward and
 * "Custom Backpropagation"; the overlap of transfers with compute is this
 * library's, the page has none.)
 * q, k, v, dout  in : host [batch, heads, n, d] bf16.
 * lengths        in : host int32 [batch] or NULL (see conventions).
 * o              out: host [batch, heads, n, d] bf16.
 * lse            out: host [batch, heads, n] fp32, or NULL when not wanted.
 * dq, dk, dv     out: host [batch, heads, n, d] bf16.
 * workspace          : DEVICE scratch of at least
 *                      nb_attn_fwd_bwd_host_workspace_size(...) bytes,
 *                      256-byte aligned, owned by the caller; contents on entry
 *                      do not matter.  It holds a few chunks at a time, not the
 *                      whole problem.
 * The work is cut into about 32 chunks: groups of whole (batch, head) slices,
 * or, when there are fewer than 32 slices, windows of one slice's sequence
 * (the rows a window owns plus 2R blocks of context on each side, which make
 * the owned rows' results exact; only those are copied back).  Chunk i + 1 is
 * copied to the device while chunk i computes on `stream` and chunk i - 1 is
 * copied back, on two streams the call creates and releases.  The host
 * buffers must be page-locked (cudaHostAlloc / cudaHostRegister) for the
 * copies to overlap; pageable memory gives the same results, serialised.
 * `lengths` is also read on the host during the call (window lengths).
 * The call is asynchronous: it returns once everything is queued, and the
 * outputs are complete when `stream` reaches the point where the call was
 * made (synchronise it before reading them).  The host inputs must stay
 * unchanged and the outputs unread until then.  Results equal those of
 * nb_attn_fwd + nb_attn_bwd on device copies of the same tensors, up to the
 * order of fp32 additions: dQ's atomic additions and, in windows, the online
 * softmax and accumulation over the same keys from another first chunk.  The
 * workspace size depends on R (through the windows' context).
 * Errors: as nb_attn_bwd (NB_BF16 only; NB_F32 returns NB_ERR_UNSUPPORTED);
 * a CUDA failure after some chunks were queued returns NB_ERR_CUDA with the
 * queued work still ordered before later work on `stream`.
 */
NB_API size_t nb_attn_fwd_bwd_host_workspace_size(int batch, int heads, int n, int d, int R,
                                                  int dtype);
NB_API nb_status nb_attn_fwd_bwd_host(const void* q, const void* k, const void* v,
                                      const void* dout, const int32_t* lengths, void* o,
                                      float* lse, void* dq, void* dk, void* dv, void* workspace,
                                      size_t workspace_bytes, int batch, int heads, int n, int d,
                                      int R, int dtype, int causal, void* stream);

/*
 * nb_attn_bwd_noalloc - nb_attn_bwd for callers that cannot allocate device
 * memory.  The NucleoByte page has no counterpart: it exists for callers that
 * cannot hand the library a workspace, such as a host program whose device
 * memory is wholly owned by another allocator, an embedding through a
 * foreign-function interface with no allocator, or a latency-critical loop in
 * which cudaMalloc/cudaFree (which may synchronise the device) are not allowed.
 * Same arguments, results and errors as nb_attn_bwd, minus the workspace: the
 * scratch is a fixed array of NB_NOALLOC_SCRATCH_BYTES compiled into the
 * library, held on every GPU where the library's code is loaded until the
 * process exits.  Shapes whose nb_attn_bwd_workspace_size exceeds that limit
 * return NB_ERR_WORKSPACE without launching.  This entry point allocates
 * nothing.  Its first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream
 * capture.  Every call shares the one array, so calls that overlap on the GPU
 * (other streams or host threads) race and must be serialised by the caller;
 * each call rewrites what it reads from the array, so an earlier call's
 * leftover contents do not affect results.
 */
#define NB_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
NB_API nb_status nb_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, const int32_t* lengths,
                                     void* dq, void* dk, void* dv, int batch, int heads, int n,
                                     int d, int R, int dtype, void* stream);

/*
 * nb_tokenize_kmer - fused 2-bit DNA k-mer tokenizer.
 * (NucleoByte page, sections 1 "Token Blur", 2 "Fused 2-Bit Tokenization",
 * 5 "Architecture Size" and "Evaluation Output Verification".)
 * seq     in : len ASCII bytes (any alignment).  A=0, C=1, G=2, T=3; any other
 *              byte is invalid.
 * ids     out: uint16 [len - k + 1] (nothing when len < k) or NULL: window p has
 *              ID sum_t code[p+t] * 4^(k-1-t) (first base most significant), or
 *              4^k when the window holds an invalid byte.
 * packed  out: uint8 [(len + 3) / 4] or NULL: 4 bases per byte, first base in
 *              bits 7..6, invalid bases stored as 0, unused tail slots 0.
 * k: 1..7 (the page uses 6).  len >= 0.  ids must be 2-byte aligned.
 * Both outputs NULL is valid and does nothing.
 */
NB_API nb_status nb_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                           int k, void* stream);

/*
 * nb_tokenize_batch - a batch of DNA sequences straight to model input IDs,
 * padded to a common length that is a multiple of 32.
 * (NucleoByte page, section 2 items 1-2 "Fused 2-Bit Tokenization" and
 * "Dynamic Ceiling Hardware Alignment"; section 5 "Architecture Size": a
 * 4096-entry 6-mer vocabulary plus padding/mask, and "Evaluation Output
 * Verification"; section 6: vocab_size 4100, input IDs drawn from 1 upward.)
 * Model IDs, for window size k:
 *   NB_PAD_ID (0)          padding past a sequence's last window;
 *   raw + 1 in [1, 4^k]    a window of valid bases (raw = the nb_tokenize_kmer ID);
 *   4^k + 1                a window holding an invalid byte;
 *   4^k + 2                the mask ID (never written here; for the caller's masking).
 * For k = 6 this is the page's vocabulary of 4100 (IDs 0..4099, 4099 unused).
 * seqs      in : the batch's bases, concatenated (any alignment).
 * offsets   in : int64 [batch + 1]: sequence b is seqs[offsets[b] .. offsets[b+1]).
 *                Offsets that decrease give an empty sequence.
 * input_ids out: int64 [batch][n_pad], 16-byte aligned.  Row b holds the model
 *                IDs of its windows (stride 1) followed by NB_PAD_ID.
 * lengths   out: int32 [batch] or NULL: the number of windows of each sequence,
 *                max(0, bases - k + 1), the attention's per-sequence length.
 * n_pad: a multiple of 32 (the dynamic ceiling: the smallest multiple of 32 that
 *        holds the longest sequence's windows); a sequence with more windows
 *        keeps its first n_pad and reports lengths[b] = n_pad.
 * k: 1..7.  batch >= 0.
 */
#define NB_PAD_ID 0
NB_API nb_status nb_tokenize_batch(const uint8_t* seqs, const int64_t* offsets, int batch, int k,
                                   int64_t* input_ids, int32_t* lengths, int n_pad, void* stream);

/*
 * nb_batch_ceiling - the dynamic ceiling of a batch for nb_tokenize_batch: the
 * smallest multiple of 32 that holds the longest sequence's k-mer windows.
 * (NucleoByte page, section 2 item 2 "Dynamic Ceiling Hardware Alignment": a
 * batch is padded only up to the next multiple of 32 above its longest
 * sequence, not to a fixed maximum length.)
 * offsets in : HOST int64 [batch + 1], the same offsets nb_tokenize_batch takes;
 *              sequence b has max(0, offsets[b+1] - offsets[b]) bases and
 *              max(0, bases - k + 1) windows.
 * n_pad   out: HOST int32; 0 for an empty batch or one without a window.
 * k: 1..7.  batch >= 0.  A ceiling above INT32_MAX returns NB_ERR_INVALID_ARG.
 * Runs on the host only (no device, no stream, no launch).
 */
NB_API nb_status nb_batch_ceiling(const int64_t* offsets, int batch, int k, int32_t* n_pad);

#ifdef __cplusplus
}
#endif

#endif /* NB_H_ */
