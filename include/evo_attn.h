/*
 * evo_attn.h — C ABI of the B200 (sm_100a) biased-attention library,
 * libevoattn.so: the forward pass, its backward pass, and the
 * triangle-multiplication contraction.
 *
 * The operation is the forward pass that the DeepSpeed DS4Sci_EvoformerAttention
 * guide (hmyw.cn) describes for the four Evoformer attention variants (its
 * section 5.3: MSA row-wise, MSA column-wise, triangle attention around the
 * starting node and around the ending node):
 *
 *     O[b,n,i,h,:] = sum_j softmax_j(t)[j] * V[b,n,j,h,:]
 *     t_j          = Q[b,n,i,h,:] . K[b,n,j,h,:] / sqrt(D)
 *                    + mask_bias[b,n,0,0,j] + pair_bias[b,0,h,i,j]
 *     LSE[b,n,h,i] = log sum_j exp(t_j)              (natural log)
 *
 * with the unified layout [*, L, Head, Dim] of its section 5.2 written out as
 * Q, K, V, O = [B, N, S, H, D], the residue-mask bias [B, N, 1, 1, S] and the
 * pair bias [B, 1, H, S, S] that is shared by every n (section 5.2), and the
 * FlashAttention-style log-sum-exp the forward kernel also returns (section
 * 5.4).  The four variants differ only in what N and S mean and in whether a
 * pair bias is passed (section 5.3); the caller lays the tensors out for the
 * variant it wants (for the ending-node case it passes the edges of the other
 * side, already transposed).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, all on one
 *    device (else EVO_ERR_INVALID_ARG).  The call runs on the device that owns
 *    Q and leaves the caller's current device as it found it.  The library
 *    keeps no reference to the pointers after the call returns and allocates
 *    nothing per call.
 *  - Tensors are dense and contiguous (row-major in the shapes above).
 *  - Calls are asynchronous on `stream` (NULL = the legacy default stream);
 *    the library never synchronises on its own.
 *  - Arguments are checked before anything is launched; a bad argument
 *    returns a negative evo_status_t and launches nothing.  The library never
 *    aborts or throws.
 *  - A kernel that stops waiting on an internal barrier after about two
 *    seconds records EVO_ERR_TIMEOUT in a device status word and exits; read
 *    it with evo_attn_sync_status().
 */
#ifndef EVO_ATTN_H
#define EVO_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EVO_API __attribute__((visibility("default")))
#else
#define EVO_API
#endif

/* Same object as cudaStream_t, declared here so that including this header
 * does not require the CUDA headers. */
typedef struct CUstream_st* evo_stream_t;

typedef enum {
    EVO_DTYPE_BF16 = 0,   /* bf16 inputs and O, fp32 arithmetic, tensor cores */
    EVO_DTYPE_FP32 = 1,   /* fp32 inputs and O, fp32 arithmetic throughout    */
    EVO_DTYPE_FP16 = 2    /* fp16 inputs and O, as EVO_DTYPE_BF16              */
} evo_dtype_t;

typedef enum {
    EVO_OK                    =  0,
    EVO_ERR_INVALID_ARG       = -1,  /* NULL pointer, negative size, overlap   */
    EVO_ERR_UNSUPPORTED_DTYPE = -2,  /* dtype not one of evo_dtype_t           */
    EVO_ERR_UNSUPPORTED_SHAPE = -3,  /* outside the supported envelope below   */
    EVO_ERR_MISALIGNED        = -4,  /* a pointer breaks the alignment rule    */
    EVO_ERR_CUDA              = -5,  /* a CUDA runtime/driver call failed      */
    EVO_ERR_TIMEOUT           = -6,  /* a device-side wait gave up (see above) */
    EVO_ERR_RANGE             = -7,  /* an input value is outside the range the
                                        kernel's arithmetic supports (see below) */
    EVO_ERR_SCRATCH           = -8   /* evo_attn_bwd_noalloc: the problem needs more
                                        scratch than the library's static array holds */
} evo_status_t;

/*
 * evo_attn_fwd — the fused forward pass.
 *
 *   Q, K, V    [B, N, S, H, D] of `dtype` (bf16, fp16 or fp32).
 *   mask_bias  [B, N, 1, 1, S] of `dtype`, or NULL for no mask bias.  The
 *              guide's tests pass it as 1e9 * (mask - 1) (section 5.2), so a
 *              masked key carries -1e9 (-998244352 once rounded to bf16).  A
 *              row whose every key is masked that way still follows the
 *              formula: the mask is then a constant shift of the row.  A row
 *              with no finite logit at all (every key -inf) returns O = 0 and
 *              LSE = -inf.
 *   pair_bias  [B, 1, H, S, S] of `dtype`, indexed [.., query i, key j], or
 *              NULL (the column-wise variant passes none, section 5.3(b)).
 *   O          [B, N, S, H, D] of `dtype`, written.
 *   LSE        [B, N, H, S] fp32, natural log, written.  (The guide's kernel
 *              pads the last axis to a multiple of 32; this one does not.)
 *   B, N, S, H >= 0 (a zero size is a no-op that returns EVO_OK and may come
 *              with NULL pointers), D >= 1.
 *   dtype      an evo_dtype_t.
 *   stream     CUDA stream the kernel is launched on.
 *
 * Supported envelope:
 *   EVO_DTYPE_BF16, D in {16, 32, 64, 128}: the tcgen05 tensor-core kernel
 *                   (fp32 accumulation in tensor memory; 3, 3, 2 and 1 n
 *                   slices per tile).  Q, K, V, O 16-byte aligned;
 *                   mask_bias 2-byte aligned; pair_bias 16-byte aligned when
 *                   S is a multiple of 8 (its rows are then loaded by the
 *                   tensor-memory accelerator), else 2-byte aligned (then
 *                   read element by element, somewhat slower).  The softmax
 *                   numerators P are rounded to fp16 for the P.V product, so
 *                   V is converted to fp16 on chip: every |V| must be
 *                   <= 65504, else the kernel records EVO_ERR_RANGE (read by
 *                   evo_attn_sync_status) and O is not valid.
 *   EVO_DTYPE_BF16, any other 1 <= D <= 128: the SIMT kernel of
 *                   EVO_DTYPE_FP32 (fp32 arithmetic from the exactly widened
 *                   bf16 inputs, O rounded to bf16), tens of times slower;
 *                   every pointer 2-byte aligned; no range limit on V.
 *   EVO_DTYPE_FP16: the same envelope, kernels and alignment as
 *                   EVO_DTYPE_BF16, with fp16 loads, biases and O (V needs
 *                   no conversion).  The guide's mask 1e9 * (mask - 1) is
 *                   -inf in fp16 (the guide notes fp16 for its own kernel,
 *                   section 3.3), so a row whose every key is masked returns
 *                   O = 0 and LSE = -inf.
 *   EVO_DTYPE_FP32: 1 <= D <= 128, any S; 4-byte alignment.  Plain fp32 FMA.
 *   Every element count must fit in int64 and the grid in CUDA's limits.
 *   O and LSE must not overlap each other or any input.
 *
 * Returns EVO_OK once the work is enqueued, or a negative evo_status_t.
 */
EVO_API int evo_attn_fwd(const void* Q, const void* K, const void* V,
                 const void* mask_bias, const void* pair_bias,
                 void* O, float* LSE,
                 int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
                 int dtype, evo_stream_t stream);

/*
 * evo_attn_fwd_host — evo_attn_fwd for inputs and outputs in page-locked
 * HOST memory, with the copies overlapped with the computation.
 *
 *   Qh, Kh, Vh, mask_h, pair_h  host inputs, same layouts as evo_attn_fwd
 *                               (mask_h / pair_h may be NULL).
 *   Oh, LSEh                    host outputs, same layouts.
 *   Qd, Kd, Vd, mask_d, pair_d, Od, LSEd
 *                               device buffers of the full sizes, owned by
 *                               the caller, used as the device side of the
 *                               call; mask_d / pair_d are NULL exactly when
 *                               mask_h / pair_h are.
 *   B, N, S, H, D, dtype        as for evo_attn_fwd.
 *   chunk_n                     n slices per chunk (>= 1), or 0 for about
 *                               eight chunks per batch entry.
 *   stream                      the call is ordered after the work already
 *                               on `stream`, and the work on `stream` after
 *                               it is ordered after its last copy back:
 *                               synchronise `stream` before reading Oh, LSEh,
 *                               and keep every host and device buffer of the
 *                               call allocated and unchanged until then (as
 *                               with cudaMemcpyAsync: the copies run later).
 *
 * The work is split into chunks of chunk_n n slices (the forward pass is
 * independent per (b, n); the pair bias of batch entry b is copied once).
 * For each chunk the library copies its inputs to the device on a copy
 * stream of its own, runs the kernel on `stream`, and copies O and LSE back
 * on a second copy stream, so the copy in of one chunk, the kernel of the
 * previous one and the copy back of the one before run at the same time.
 * The two copy streams and a few events are created once per device, on
 * the first call, and kept; concurrent calls on one device are enqueued one
 * after the other.  Host pointers must be page-locked (cudaHostAlloc or
 * cudaHostRegister), else EVO_ERR_INVALID_ARG; the device buffers get every
 * check of evo_attn_fwd, with the same status codes.
 */
EVO_API int evo_attn_fwd_host(const void* Qh, const void* Kh, const void* Vh, const void* mask_h,
                      const void* pair_h, void* Oh, float* LSEh,
                      void* Qd, void* Kd, void* Vd, void* mask_d, void* pair_d, void* Od, float* LSEd,
                      int64_t B, int64_t N, int64_t S, int64_t H, int64_t D, int dtype, int64_t chunk_n,
                      evo_stream_t stream);

/*
 * evo_attn_bwd_workspace_size — bytes of device workspace evo_attn_bwd needs
 * for these sizes (the same for every dtype and for every choice of
 * requested bias gradients), or a negative evo_status_t for negative sizes
 * (EVO_ERR_INVALID_ARG) or sizes whose byte counts overflow int64
 * (EVO_ERR_UNSUPPORTED_SHAPE).
 */
EVO_API int64_t evo_attn_bwd_workspace_size(int64_t B, int64_t N, int64_t S, int64_t H, int64_t D);

/*
 * evo_attn_bwd — the backward pass: gradients of a loss with respect to the
 * inputs of evo_attn_fwd, given the gradient dO with respect to O.
 *
 * The guide (sections 1 and 5.4) describes the backward kernel of its
 * FlashAttention-style design: it does not keep the S x S attention weights
 * of the forward pass but recomputes them from Q, K, V, O and the forward's
 * log-sum-exp, with the per-row delta = dO . O as an intermediate, and it
 * computes the gradient of a bias only when the caller needs it.  The guide
 * gives no formula; the gradients are the chain rule of the forward formula
 * above.  Per (b, n, h) slice, with p_ij the softmax weights and
 * dt_ij = p_ij (dO_i . V_j - delta_i) the gradient of the logit t_ij:
 *     dQ_i = sum_j dt_ij K_j / sqrt(D),   dK_j = sum_i dt_ij Q_i / sqrt(D),
 *     dV_j = sum_i p_ij dO_i,
 *     dmask[b,n,0,0,j] = sum_h sum_i dt_ij    (the mask is shared by heads and rows),
 *     dpair[b,0,h,i,j] = sum_n dt_ij          (the pair bias is shared by every n).
 *
 *   Q, K, V, mask_bias, pair_bias, dtype, B, N, S, H, D
 *              as passed to evo_attn_fwd (same layouts and NULL rules).
 *   O, LSE     the outputs of evo_attn_fwd for exactly those inputs.
 *   dO         [B, N, S, H, D] of `dtype`: the gradient with respect to O.
 *   dQ, dK, dV [B, N, S, H, D] of `dtype`, written.
 *   dmask      [B, N, 1, 1, S] of `dtype`, written, or NULL to skip this
 *              gradient (NULL is required when mask_bias is NULL).
 *   dpair      [B, 1, H, S, S] of `dtype`, written, or NULL to skip this
 *              gradient (NULL is required when pair_bias is NULL).
 *   workspace  device scratch of at least evo_attn_bwd_workspace_size(B, N,
 *              S, H, D) bytes (workspace_bytes says how many), 256-byte
 *              aligned, owned by the caller; its contents on entry do not
 *              matter and are overwritten.  Keep it allocated and do not use
 *              it for anything else until the call's work on `stream` is done.
 *   stream     CUDA stream the kernels are launched on.
 *
 * A row whose every key carries the guide's -1e9 mask follows the formula
 * (the mask is a constant shift of the row, as in the forward pass); its
 * row statistics are then recomputed from the inputs, because the fp32 LSE
 * near -1e9 has lost the digits that matter.  A row with no finite logit
 * (every key -inf) has no weights and contributes zero to every gradient.
 *
 * Supported envelope: every dtype, 1 <= D <= 128, any S; pointers aligned to
 * the element size (LSE to 4 bytes).  Two implementations:
 *   - tcgen05 tensor cores for EVO_DTYPE_BF16 / EVO_DTYPE_FP16 with D in
 *     {16, 32, 64}, no pair bias or S a multiple of 8, and Q, K, V, dO, dQ,
 *     dK, dV (and the pair bias) 16-byte aligned: S, dP, dV, dK and dQ are
 *     MMAs with fp32 accumulation; the weights p and logit gradients dt
 *     enter them rounded to the input type; dQ, dmask and dpair are summed
 *     in fp32 in the workspace (with atomic adds, so the order of the
 *     additions, and the last bits of those three gradients, can vary from
 *     call to call) and rounded at the end;
 *   - plain fp32 FMA arithmetic for every other accepted call (fp32 inputs,
 *     other head dims, pair-bias rows that are not 16-byte units, less
 *     aligned pointers), recomputing the weights per gradient; deterministic,
 *     and far slower.
 * The gradients of a call are computed by several kernels (and zeroing
 * copies) on `stream` and are complete once its work there is.  Outputs and
 * workspace must not overlap each other or any input.
 *
 * Returns EVO_OK once the work is enqueued, or a negative evo_status_t
 * (EVO_ERR_INVALID_ARG also for a workspace that is too small, or a gradient
 * of a bias that was not passed).
 */
EVO_API int evo_attn_bwd(const void* Q, const void* K, const void* V,
                 const void* mask_bias, const void* pair_bias,
                 const void* O, const float* LSE, const void* dO,
                 void* dQ, void* dK, void* dV, void* dmask, void* dpair,
                 void* workspace, int64_t workspace_bytes,
                 int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
                 int dtype, evo_stream_t stream);

/*
 * evo_attn_bwd_noalloc — evo_attn_bwd without a caller workspace: the
 * scratch is a static array of EVO_ATTN_NOALLOC_SCRATCH_BYTES (64 MiB) per
 * device inside this library, so the call allocates no memory of any kind.
 * The guide has no counterpart; this is an interface of this library.
 *
 * For callers that cannot allocate device memory at the point of the call:
 * a process that has handed all of the device's memory to a pool of its own
 * (so that a new allocation would fail or fragment it), or code that must
 * not bring in the device-wide synchronisation that releasing device memory
 * (cudaFree) implies.  Everything else is as for evo_attn_bwd (arguments
 * without workspace / workspace_bytes, envelope, status codes, gradients).
 *
 *  - Size limit: evo_attn_bwd_workspace_size(B, N, S, H, D) must not exceed
 *    EVO_ATTN_NOALLOC_SCRATCH_BYTES, else EVO_ERR_SCRATCH is returned and
 *    nothing is launched (e.g. B=1, N=64, S=256, H=4, D=32 needs 10.0 MB;
 *    N=S=384, H=4, D=32 needs 83 MB and is refused).
 *  - Setup: the first call on a device looks up the array's device address
 *    (once per device, with that device current) and keeps it; make that
 *    first call before any stream capture on the device.
 *  - Zeroing: the call itself clears, on `stream`, the parts of the scratch
 *    that must start at zero (the fp32 sums of dQ, dmask and dpair and a
 *    work-list counter); no other part needs to start at zero, and nothing
 *    of one call is read by the next.
 *  - Concurrency: every call on a device uses the same array.  Calls whose
 *    work overlaps on the device (on different streams without ordering
 *    between them, or from several host threads) race on it and give wrong
 *    gradients; order them (one stream, or events).
 */
#define EVO_ATTN_NOALLOC_SCRATCH_BYTES (64ll << 20)
EVO_API int evo_attn_bwd_noalloc(const void* Q, const void* K, const void* V,
                 const void* mask_bias, const void* pair_bias,
                 const void* O, const float* LSE, const void* dO,
                 void* dQ, void* dK, void* dV, void* dmask, void* dpair,
                 int64_t B, int64_t N, int64_t S, int64_t H, int64_t D,
                 int dtype, evo_stream_t stream);

/*
 * evo_trimul_workspace_size — bytes of device workspace evo_trimul needs
 * (three [Bt*C, N, Np] copies, Np = N rounded up to a multiple of 8), or a
 * negative evo_status_t for negative sizes or byte counts past int64.
 */
EVO_API int64_t evo_trimul_workspace_size(int64_t Bt, int64_t N, int64_t C);

/*
 * evo_trimul — triangle multiplication: the contraction over the third node
 * of two edge representations, channel by channel.
 *
 * The NVIDIA cuEquivariance blog (open-lab.net, "Accelerated molecular
 * modeling with NVIDIA cuEquivariance and NVIDIA NIM microservices", the
 * triangle-operations sections) names triangle multiplication beside
 * triangle attention as the two O(N^3) operations of these models, from
 * "triangular relationships" (i close to k and k close to j relate i and j),
 * without a formula.  This library's reading, for every b and channel c:
 *     outgoing (outgoing = 1):  Z[b,i,j,c] = sum_k A[b,i,k,c] * B[b,j,k,c]
 *     incoming (outgoing = 0):  Z[b,i,j,c] = sum_k A[b,k,i,c] * B[b,k,j,c]
 * (the projections, gates and norms around it in a model are per-edge and
 * not part of this call).
 *
 *   A, B       [Bt, N, N, C] of `dtype`, contiguous, 2-byte aligned.
 *   Z          [Bt, N, N, C] of `dtype`, written (fp32 accumulation, rounded
 *              to nearest even); must not overlap A, B or the workspace.
 *   workspace  device scratch of at least evo_trimul_workspace_size(Bt, N, C)
 *              bytes, 256-byte aligned, owned by the caller, overwritten.
 *   Bt, N, C   >= 0 (a zero size is a no-op that returns EVO_OK).
 *   dtype      EVO_DTYPE_BF16 or EVO_DTYPE_FP16 (else EVO_ERR_UNSUPPORTED_DTYPE).
 *   stream     CUDA stream of the call.
 *
 * Three kernels on `stream`: A and B transposed to channel-first copies in
 * the workspace, a tcgen05 batched GEMM over the Bt*C channel matrices, and
 * the result transposed back.  Returns EVO_OK once enqueued, or a negative
 * evo_status_t (EVO_ERR_INVALID_ARG also for a workspace that is too small).
 * The pages have no interface for this operation; the call follows the shape
 * conventions of evo_attn_fwd.
 */
EVO_API int evo_trimul(const void* A, const void* B, void* Z, void* workspace, int64_t workspace_bytes,
               int64_t Bt, int64_t N, int64_t C, int outgoing, int dtype, evo_stream_t stream);

/*
 * evo_attn_sync_status — synchronise `stream`, then return and clear the
 * device status word of the stream's device (for the legacy default stream,
 * NULL: the current device), whichever device is current when it is called;
 * the caller's current device is left as it was.  Returns EVO_OK,
 * EVO_ERR_TIMEOUT if a kernel on that device gave up waiting since the last
 * call, EVO_ERR_RANGE if a kernel met an out-of-range input, or EVO_ERR_CUDA
 * if the stream itself reports an error.  The first error recorded since the
 * last call is the one returned.
 */
EVO_API int evo_attn_sync_status(evo_stream_t stream);

/*
 * evo_attn_selftest_timeout — exercises the device-side failure path without
 * faulting anything: launches one warp on `stream` that waits on an internal
 * barrier that nothing ever completes, with a limit of `limit_ns`
 * nanoseconds (1 .. 1e9).  The wait gives up, records EVO_ERR_TIMEOUT in the
 * status word and the kernel ends normally; *result (a device int) is set to
 * 0.  A following evo_attn_sync_status(stream) returns EVO_ERR_TIMEOUT and
 * clears the word.  The guide has no counterpart; this is a diagnostic of this
 * library's bounded waits.  Returns EVO_OK once launched, EVO_ERR_INVALID_ARG
 * for a limit outside the range or a NULL / non-device result pointer.
 */
EVO_API int evo_attn_selftest_timeout(int64_t limit_ns, int* result, evo_stream_t stream);

/* evo_attn_strerror — a static, human-readable string for a status code. */
EVO_API const char* evo_attn_strerror(int status);

/* evo_attn_version — library version as major*10000 + minor*100 + patch. */
EVO_API int evo_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EVO_ATTN_H */
