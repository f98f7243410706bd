/*
 * fa2.h -- C ABI of libfa2.so: FlashAttention-2 style (causal) multi-head
 * attention forward and recomputation backward for NVIDIA B200 (sm_100a).
 *
 * The operation (CS336 A2 Systems handout, section 4.2.2):
 *   forward   S = scale * Q K^T                       (Eq. 4; scale = 1/sqrt(d)
 *                                                      in the handout)
 *             causal: key j is visible to query i iff j <= i
 *                                                     (Problem flash_forward (c))
 *             P = softmax_row(S), O = P V             (Eqs. 5-6)
 *             L_i = log sum_j exp(S_ij)               (Eq. 12, natural log)
 *             computed tile by tile with the online softmax of Algorithm 1.
 *   backward  D_i = rowsum(O o dO)_i                  ("backward pass with
 *                                                      recomputation")
 *             P_ij = exp(S_ij - L_i), dV = P^T dO, dP = dO V^T,
 *             dS_ij = P_ij (dP_ij - D_i), dQ = scale dS K, dK = scale dS^T Q
 *                                                     (Eqs. 13-19)
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, contiguous, row-major [B, H, N, d] arrays in device
 *     memory (q, k, v, o, dout, dq, dk, dv), in the element type `dtype`.
 *     lse is a dense [B, H, N] float32 device array (natural log).
 *   - Supported: B >= 1, H >= 1, 1 <= N <= 2^24, d in {16, 32, 64, 80, 128}.
 *     N need not be a multiple of any tile size.
 *   - Tensor pointers must be 16-byte aligned (they are read and written by
 *     the tensor memory accelerator); lse must be 4-byte aligned; the
 *     backward workspace must be 256-byte aligned.
 *   - The caller owns every buffer.  The library never allocates or frees
 *     device memory and keeps no pointer after a call returns.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Calls are asynchronous and never synchronise the host.
 *   - Arguments are validated on the host before anything is enqueued; on a
 *     validation error nothing is launched and the outputs are untouched.
 *   - A device-side pipeline watchdog bounds every wait inside the kernels.
 *     If one expires, the kernel stops early, leaves its outputs undefined
 *     and records FA2_ERR_DEVICE_TIMEOUT in a per-device status word that
 *     fa2_last_device_status() reads once the caller has synchronised.
 *   - Thread safety: entry points may be called concurrently from several
 *     host threads; the only shared host state is a mutex-guarded cache of
 *     per-device kernel attributes and of the device addresses of the
 *     library's own device variables (the status word, the scratch array of
 *     fa2_backward_noalloc), looked up once per device.  A device reset
 *     (cudaDeviceReset) invalidates those addresses: the library is not
 *     usable on that device afterwards in the same process.
 */
#ifndef FA2_H_
#define FA2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of q, k, v, o, dout, dq, dk, dv.  Accumulation is always fp32.
 * FA2_FP32 inputs are consumed by the tensor cores as TF32 (rounded to
 * nearest); FA2_BF16 and FA2_FP16 inputs directly, with P and dS rounded to
 * the input type before their MMAs. */
typedef enum {
    FA2_BF16 = 0,
    FA2_FP32 = 1,
    FA2_FP16 = 2
} fa2_dtype;

typedef enum {
    FA2_OK = 0,
    FA2_ERR_NULL_PTR = 1,             /* a required pointer is NULL                */
    FA2_ERR_BAD_SHAPE = 2,            /* B, H or N out of range                    */
    FA2_ERR_UNSUPPORTED_HEAD_DIM = 3, /* d not in {16, 32, 64, 80, 128}            */
    FA2_ERR_UNSUPPORTED_DTYPE = 4,    /* dtype not a fa2_dtype value               */
    FA2_ERR_MISALIGNED = 5,           /* a pointer breaks the alignment rules      */
    FA2_ERR_WORKSPACE_TOO_SMALL = 6,  /* workspace_bytes < fa2_backward_workspace_bytes */
    FA2_ERR_CUDA = 7,                 /* a CUDA runtime/driver call or launch failed */
    FA2_ERR_DEVICE_TIMEOUT = 8,       /* a kernel's pipeline watchdog expired      */
    FA2_ERR_UNSUPPORTED_DEVICE = 9,   /* the current device is not sm_100          */
    FA2_ERR_BAD_ARGUMENT = 10,        /* scale not finite and > 0, causal not 0/1,
                                         watchdog self-test limit out of range     */
    FA2_ERR_SCRATCH_TOO_SMALL = 11    /* problem too big for fa2_backward_noalloc  */
} fa2_status;

/* Opaque CUDA stream handle; identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* fa2_stream_t;

/*
 * Forward pass (handout section 4.2.2, Algorithm 1 with the causal rule of
 * Problem flash_forward (c)).
 *   q, k, v  in : [B, H, N, d] `dtype`
 *   o        out: [B, H, N, d] `dtype`, O = softmax(scale Q K^T (+mask)) V,
 *                 rounded once from fp32
 *   lse      out: [B, H, N] float32, L_i = log sum_j exp(S_ij)
 *   causal   1 = causal mask, 0 = full attention
 *   scale    finite, positive multiplier of Q K^T (1/sqrt(d) in the handout)
 * Returns FA2_OK once the work is enqueued, or a validation / launch error.
 */
fa2_status fa2_forward(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int N, int d, int causal, float scale,
                       fa2_dtype dtype, fa2_stream_t stream);

/*
 * The general forward: grouped-query attention and different query and key
 * lengths.
 *   - H query heads share H_kv key/value heads (the "LLM FLOPs Computation"
 *     page, section Extension: GQA): query head h of a batch uses key/value
 *     head h / (H / H_kv); H_kv = H is multi-head, H_kv = 1 multi-query
 *     attention.  H must be a multiple of H_kv.
 *   - N query rows attend to Nk key/value rows (the handout's Algorithm 1
 *     takes N_q and N_k separately, section 4.2.2).  With causal = 1 key j is
 *     visible to query i iff j <= i (the same index comparison as for
 *     N_q = N_k), so keys at or past N are seen by no query.
 *   q, o   [B, H, N, d];  k, v  [B, H_kv, Nk, d];  lse [B, H, N] float32
 * fa2_forward(...) is fa2_forward_ex(..., H_kv = H, N, Nk = N, ...).  Shapes
 * out of range (H not a multiple of H_kv, Nk < 1 or > 2^24) give
 * FA2_ERR_BAD_SHAPE; otherwise as fa2_forward.
 */
fa2_status fa2_forward_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                          fa2_dtype dtype, fa2_stream_t stream);

/*
 * Bytes of device workspace fa2_backward needs for these sizes: the fp32 D
 * and log2-scaled L vectors, 2 * 4 * B * H * ceil(N / 128) * 128 bytes; for
 * 16-bit inputs with N > 128 (where the one-pass form of fa2_backward_opts
 * can run) also the fp32 dQ accumulator, 4 * B * H * ceil(N / 128) * 128 * d bytes; for FA2_FP32 instead
 * copies of q, k, v and dout rounded to TF32 (round to nearest),
 * 4 * 4 * B * H * N * d bytes (every region rounded up to 256 bytes).
 * Returns 0 for arguments fa2_backward would reject.
 */
size_t fa2_backward_workspace_bytes(int B, int H, int N, int d, fa2_dtype dtype);

/*
 * Workspace of fa2_backward_ex: as fa2_backward_workspace_bytes, except that
 * the FA2_FP32 copies of k and v have B * H_kv * Nk * d elements, and that for
 * 16-bit inputs with few key/value tiles (ceil(Nk / 128) * B * H_kv < 148 and
 * H_kv < H) the dK/dV pass splits each query-head group over S =
 * min(H / H_kv, ceil(296 / (ceil(Nk / 128) * B * H_kv))) thread blocks whose
 * fp32 partial dK and dV, 2 * S * B * H_kv * ceil(Nk / 128) * 128 * d * 4
 * bytes, are summed in a fixed order afterwards (such problems take the
 * two-pass form and need no dQ accumulator).  Returns 0 for arguments
 * fa2_backward_ex would reject.
 */
size_t fa2_backward_workspace_bytes_ex(int B, int H, int H_kv, int N, int Nk, int d,
                                       fa2_dtype dtype);

/*
 * Backward pass with recomputation (handout section 4.2.2, Eqs. 13-19;
 * D = rowsum(O o dO)), organised as the handout's Algorithm 2 (section
 * 4.2.3): one pass over query tiles recomputes P and accumulates dQ, a second
 * pass over key/value tiles accumulates dK and dV, so nothing is added across
 * thread blocks.  Rows of a query tile that sees a single key tile (causal:
 * the first 128 rows) take D in its equivalent form sum_j P_ij dP_ij from the
 * recomputed P and dP, and their dS enters the dQ and dK contractions as two
 * 16-bit parts (hi + lo); these rows see few keys, so |dS| is of the order of
 * |dP| and D from the rounded O would not be accurate enough.
 *   q, k, v, o, dout  in : [B, H, N, d] `dtype` (o as produced by fa2_forward)
 *   lse               in : [B, H, N] float32 from fa2_forward
 *   dq, dk, dv        out: [B, H, N, d] `dtype`
 *   workspace         scratch of at least fa2_backward_workspace_bytes bytes,
 *                     256-byte aligned, owned by the caller; its contents on
 *                     entry do not matter and on return are unspecified
 * This is fa2_backward_opts with flags = 0 (the two-pass form: every output
 * is bitwise reproducible); fa2_backward_opts with FA2_BWD_ONE_PASS selects
 * the one-pass form.
 */
fa2_status fa2_backward(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, void* dq, void* dk, void* dv,
                        int B, int H, int N, int d, int causal, float scale, fa2_dtype dtype,
                        void* workspace, size_t workspace_bytes, fa2_stream_t stream);

/*
 * Backward pass of fa2_forward_ex: dq [B, H, N, d]; dk, dv [B, H_kv, Nk, d],
 * each key/value head's gradient being the sum over the H / H_kv query heads
 * that share it (accumulated in one thread block, so still deterministic);
 * key rows no query sees get zero gradients.  The workspace is
 * fa2_backward_workspace_bytes_ex(B, H, H_kv, N, Nk, d, dtype) bytes.  Other
 * arguments, results and errors are those of fa2_backward.
 */
fa2_status fa2_backward_ex(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, void* dq, void* dk, void* dv,
                           int B, int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                           fa2_dtype dtype, void* workspace, size_t workspace_bytes,
                           fa2_stream_t stream);

/*
 * Block-sparse attention ("Notes on flashattention" post, section
 * "Block-sparse Flashattention", Proposition 4): blocks of 128 query rows by
 * 128 key rows whose mask byte is 0 are skipped; their scores take no part in
 * the softmax.
 *   block_mask  in : DEVICE pointer to ceil(N / 128) * ceil(Nk / 128) bytes,
 *                    row-major (one row per 128-row query tile); entry (a, b)
 *                    nonzero lets query rows [128a, 128a + 128) attend to key
 *                    rows [128b, 128b + 128).  One mask for every batch and
 *                    head; owned by the caller, read by the kernels only.
 * With causal = 1 key j is visible to query i iff j <= i and its block is set.
 * A query row that sees no key (its block row is empty) gets O = 0 and
 * L = -inf; its dQ is 0 and it adds nothing to dK or dV.  Other arguments,
 * results and the workspace are those of fa2_forward_ex / fa2_backward_ex.
 * Every input type and any N and Nk the dense calls accept (a thread block
 * keeps the tiles it visits in a list of 512 entries, 16-bit inputs, and walks
 * the mask itself past that or for fp32 inputs).  Errors: block_mask NULL ->
 * FA2_ERR_NULL_PTR.  A mask of all ones gives the results of fa2_forward_ex /
 * fa2_backward_ex.
 */
fa2_status fa2_forward_block_sparse(const void* q, const void* k, const void* v, void* o,
                                    float* lse, int B, int H, int H_kv, int N, int Nk, int d,
                                    int causal, float scale, fa2_dtype dtype,
                                    const uint8_t* block_mask, fa2_stream_t stream);

fa2_status fa2_backward_block_sparse(const void* q, const void* k, const void* v, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk,
                                     void* dv, int B, int H, int H_kv, int N, int Nk, int d,
                                     int causal, float scale, fa2_dtype dtype,
                                     const uint8_t* block_mask, void* workspace,
                                     size_t workspace_bytes, fa2_stream_t stream);

/* Flags of fa2_backward_opts. */
#define FA2_BWD_DETERMINISTIC 1u
#define FA2_BWD_ONE_PASS 2u

/*
 * The backward pass with a choice of organisation; fa2_backward,
 * fa2_backward_ex and fa2_backward_block_sparse are this entry point with
 * flags = 0.
 *
 * FA2_BWD_DETERMINISTIC: the two-pass form described at fa2_backward (the
 *   handout's Algorithm 2, section 4.2.3): every output bitwise reproducible.
 * FA2_BWD_ONE_PASS: where it applies -- 16-bit inputs, no block mask, more
 *   than one key tile (Nk > 128), and dK/dV work not split across thread
 *   blocks (see fa2_backward_workspace_bytes_ex) -- ONE pass over key/value
 *   tiles (the FlashAttention-2 backward with the key/value tile outermost,
 *   handout section 4.2.2): P, dP and dS are computed once per (key tile,
 *   query tile) pair, and each key tile's contribution scale * dS K to dQ is
 *   added into an fp32 accumulator in the workspace with TMA reduce-add; a
 *   last kernel rounds dQ once.  dK and dV are bitwise reproducible (and
 *   equal to the two-pass form's); the BITS OF dQ DEPEND ON THE ORDER in which
 *   key tiles' contributions arrive and can change from run to run (the
 *   result stays within the same tolerance).  Query tiles whose rows see a
 *   single key tile (causal: the first 128 rows) take their dQ and D from the
 *   two-pass form's query-tile pass.  Where the one-pass form does not apply,
 *   the two-pass form runs.
 * 0: currently the two-pass form.
 * Both bits together, or any other bit, give FA2_ERR_BAD_ARGUMENT.
 * block_mask: NULL, or the block mask of fa2_backward_block_sparse.
 * workspace: fa2_backward_workspace_bytes_ex(...) bytes, which covers both
 *   forms; the two-pass form also accepts the same size without the dQ
 *   accumulator (4 * B * H * ceil(N / 128) * 128 * d bytes, rounded up to 256).
 */
fa2_status fa2_backward_opts(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             int B, int H, int H_kv, int N, int Nk, int d, int causal, float scale,
                             fa2_dtype dtype, const uint8_t* block_mask, unsigned flags,
                             void* workspace, size_t workspace_bytes, fa2_stream_t stream);

/*
 * fa2_backward plus timing hooks, for profiling: identical arguments and
 * behaviour, and additionally records the caller's CUDA events (cudaEvent_t
 * handles created on the current device; any entry may be NULL) on `stream`
 * at the boundaries of the kernels the backward enqueues:
 *   events[0] before the D / L pre-pass,   events[1] after it,
 *   events[2] after the pass over query tiles (two-pass form: the dQ pass;
 *             one-pass form: that pass on the single-tile query tiles),
 *   events[3] after the pass over key tiles (the one-pass form then enqueues
 *             one more kernel, which rounds dQ).
 * `events` itself may be NULL (then this is fa2_backward).  The library only
 * records the events; the caller owns and destroys them.
 */
fa2_status fa2_backward_timed(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dout, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, int causal, float scale,
                              fa2_dtype dtype, void* workspace, size_t workspace_bytes,
                              fa2_stream_t stream, void* const* events);

/*
 * fa2_backward_noalloc -- the backward pass for callers that cannot allocate
 * device memory.  (Not part of the method the handout describes; it has no
 * counterpart there.)
 *
 * Who needs it: code that is handed only its input and output buffers and has
 * no allocator of its own -- for example a plugin running inside an inference
 * or training engine whose memory pool owns all of the GPU's memory, or a hot
 * path that must not call cudaMalloc because it would synchronise the device
 * or fragment a fully reserved heap.  Such a caller cannot provide the
 * workspace fa2_backward asks for.
 *
 * Arguments and results are those of fa2_backward without the workspace: the
 * scratch (the workspace fa2_backward_workspace_bytes sizes) lives in a fixed 64 MiB
 * array that the library places in device memory of every GPU that loads it,
 * held until the process exits.  Problems whose workspace would exceed it
 * (fa2_backward_workspace_bytes(...) > 64 MiB: for FA2_BF16, B*H*ceil(N/128)*128
 * above about 8.3 million rows; for FA2_FP32, whose workspace also holds the
 * rounded operand copies, B*H*N*d above about 4 million elements) are
 * rejected with FA2_ERR_SCRATCH_TOO_SMALL before anything is enqueued.  The call allocates nothing: no cudaMalloc,
 * cudaFree, or allocating library routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The address is kept for the life of the
 * process: after cudaDeviceReset on a device (which frees the array with the
 * context) this entry point must not be called on that device again.  Every call on a device shares the one array:
 * the kernels re-initialise all of it that must start from zero, but two
 * calls whose work overlaps on the GPU (different streams, no ordering
 * between them) race on it and give wrong results.  Order such calls on one
 * stream or with events.
 */
fa2_status fa2_backward_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk,
                                void* dv, int B, int H, int N, int d, int causal, float scale,
                                fa2_dtype dtype, fa2_stream_t stream);

/*
 * Status recorded by the kernels on the current device since the last call
 * of fa2_clear_device_status (FA2_OK or FA2_ERR_DEVICE_TIMEOUT).  Call it
 * after synchronising the streams the kernels ran on.  Returns FA2_ERR_CUDA
 * if the status word cannot be read.
 */
fa2_status fa2_last_device_status(void);

/* Reset the current device's status word to FA2_OK (synchronous). */
fa2_status fa2_clear_device_status(void);

/* Static, human-readable name of a status code. */
const char* fa2_status_string(fa2_status status);

/*
 * fa2_watchdog_selftest -- checks, on the current device, the pipeline
 * watchdog every kernel wait relies on.  (Not part of the method; it tests
 * this library's failure detection.)
 *
 * Enqueues on `stream` one warp whose first thread waits, with the kernels'
 * bounded wait, on an mbarrier that no thread ever arrives on.  The wait ends
 * after `limit_ns` nanoseconds (1e3 <= limit_ns <= 1e10, else
 * FA2_ERR_BAD_ARGUMENT) and records FA2_ERR_DEVICE_TIMEOUT in the device's
 * status word, exactly as an expired wait in an attention kernel does.  No
 * memory is read or written besides the status word; the GPU context stays
 * usable.  After synchronising `stream`, fa2_last_device_status() returns
 * FA2_ERR_DEVICE_TIMEOUT (unless an earlier error is already recorded);
 * fa2_clear_device_status() resets it.  Returns FA2_OK once enqueued, or a
 * validation / launch error.
 */
fa2_status fa2_watchdog_selftest(unsigned long long limit_ns, fa2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA2_H_ */
