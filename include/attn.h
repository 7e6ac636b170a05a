/*
 * attn.h -- C ABI of libattn_sm100.so: fused scaled-dot-product attention
 * forward pass for NVIDIA B200 (sm_100a).
 *
 * The operation (exact attention; "FlashAttention-3" explainer, droidorbit.com,
 * opening definition Softmax(Q K^T / sqrt(d)) V, with `scale` in place of
 * 1/sqrt(d); causal masking as in "FlashAttention-3: como exprimir H100 al
 * limite con atencion IO-aware", dibro.site, "Contribuciones clave"):
 *
 *   for every batch b, head h and query row i:
 *     s_ij  = scale * <Q[b,h,i,:], K[b,h,j,:]>,  j in J_i
 *     J_i   = {0 .. N-1}, or {0 .. i} when causal (queries and keys aligned)
 *     O[b,h,i,:] = sum_j softmax_j(s_i.) V[b,h,j,:]
 *     LSE[b,h,i] = ln sum_{j in J_i} exp(s_ij)
 *
 * computed tiled with online-softmax statistics (running max m, running sum
 * l; dibro.site "Arquitectura y metodo"; droidorbit.com "Mathematical
 * Formulation: The Online Softmax Rescaling Trick") so that the N x N score
 * matrix is never written to device memory.
 *
 * Conventions common to every entry point
 * ---------------------------------------
 *  - Layout: every tensor is contiguous row-major [B][H][N][d] (head dim
 *    innermost, the (batch, head, sequence, dim) stride order of the pages'
 *    kernel signature); LSE is contiguous [B][H][N] fp32, natural log.
 *  - Pointers are DEVICE pointers on the current CUDA device, 16-byte aligned
 *    (TMA requirement).  The caller owns every buffer; the library never
 *    frees or keeps them.  Outputs must not alias inputs.
 *  - The library allocates no per-call device memory.  On first use of a
 *    device it allocates one 16-byte status word (kept until exit).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous: they validate, enqueue and return.
 *  - Validation happens before any launch; on failure nothing is enqueued and
 *    the call returns ATTN_ERR_INVALID_ARG / ATTN_ERR_UNSUPPORTED /
 *    ATTN_ERR_MISALIGNED.  Launch failures return ATTN_ERR_CUDA.  No C++
 *    exception, abort or device trap crosses this boundary.
 *  - Every internal wait of the kernels is bounded (default 1 s, environment
 *    variable ATTN_WAIT_LIMIT_MS).  A wait that runs out makes the kernel
 *    record ATTN_ERR_TIMEOUT in the device status word and return; read it
 *    with attn_last_status().
 *  - Results are deterministic: the same inputs give bit-identical outputs.
 */
#ifndef ATTN_SM100_H_
#define ATTN_SM100_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* null pointer, size < 1, overflow, bad scale  */
  ATTN_ERR_UNSUPPORTED = 2,  /* head dim or dtype the library does not handle */
  ATTN_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned             */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed          */
  ATTN_ERR_TIMEOUT = 5,      /* a kernel wait ran out (read after sync)       */
  ATTN_ERR_BOUNDS = 6        /* debug build only: a TMEM or shared-memory
                                range check failed (read after sync)          */
} attn_status_t;

typedef enum {
  ATTN_BF16 = 0,
  ATTN_FP16 = 1
} attn_dtype_t;

/*
 * attn_fwd -- 16-bit attention forward.
 *   q, k, v : [B][H][N][d] bf16 or fp16 (per `dtype`), read only.
 *   o       : [B][H][N][d] same dtype, written.
 *   lse     : [B][H][N] fp32, written; may be NULL (then not written).
 *   B, H, N : >= 1, B*H*N < 2^31.
 *   d       : a multiple of 8, at most 256.  64, 128 and 256 run natively;
 *             other sizes run zero-padded to the next of those (the padding
 *             adds zero terms to every score and is never stored).
 *   scale   : finite and > 0 (usually 1/sqrt(d)).
 *   causal  : 0 or 1 (key j visible to query i iff j <= i).
 * Rounding: scores, statistics and accumulation are fp32; P is rounded to
 * the input dtype before the P.V product; O is rounded to the input dtype.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int N, int d, float scale, int causal, int dtype,
                       void* stream);

/*
 * attn_fwd_strided -- attn_fwd over strided views.  The pages' kernel
 * signature takes (batch, head, sequence) strides for Q, K, V and the output
 * ("FlashAttention-3 warp specialization on Hopper", vikram-blog.pages.dev,
 * "Production Implementation & Code Pattern"); this entry point does the
 * same, so e.g. [B][N][H][d] (BSHD) tensors need no copy.
 *   x_strides : 3 element strides of tensor x over (batch, head, row), host
 *               array; the head dim is contiguous.  Each stride must be a
 *               positive multiple of 8 elements (16 bytes) and the row
 *               stride at least d.  O's rows must not overlap one another.
 *   Everything else as attn_fwd (lse stays contiguous [B][H][N]).
 */
attn_status_t attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int N, int d, const long long* q_strides,
                               const long long* k_strides, const long long* v_strides,
                               const long long* o_strides, float scale, int causal, int dtype,
                               void* stream);

/*
 * attn_quant_fp8 -- per-block e4m3 quantisation with optional incoherent
 * processing (quantum-bit repost "H100 utilisation 75% ... FlashAttention-3",
 * third technical upgrade: block-wise quantisation and incoherent processing;
 * "FlashAttention-3 (HE)", systems-analysis.info, "Technical innovations"
 * item 3: rotate Q and K by a random orthogonal, e.g. Hadamard, matrix
 * before quantising; QK^T is unchanged).
 *   x       : [B][H][N][d] bf16 input, read only.
 *   x8      : [B][H][N][d] e4m3fn codes (uint8), written.
 *   descale : [B][H][ceil(N/128)] fp32, written: one factor per block of 128
 *             rows x d of one (b, h); x ~= value(code) * descale.
 *   hadamard: 0 = plain; 1 = rotate each row by R = diag(signs) H_d / sqrt(d)
 *             (Sylvester H_d) before quantising.  Use it for Q and K only.
 *   signs   : d fp32 values of +-1 (device pointer), or NULL for all +1.
 *             Ignored when hadamard = 0.  Q and K must use the same signs.
 *   d       : 64, 128 or 256 (others -> ATTN_ERR_UNSUPPORTED).
 * Per block: amax = max |y|; s = amax / 448 in fp32 (s = 1 if amax = 0);
 * code = e4m3_rn_satfinite(y / s) with an IEEE fp32 division.
 */
attn_status_t attn_quant_fp8(const void* x, void* x8, float* descale, int B, int H, int N,
                             int d, int hadamard, const float* signs, void* stream);

/*
 * attn_fwd_fp8 -- e4m3 attention forward (dibro.site "Arquitectura y metodo":
 * FP8 attention with in-line per-block quantisation; quantum-bit repost,
 * FP8 paragraph).
 *   q8, k8, v8 : [B][H][N][d] e4m3fn codes from attn_quant_fp8 (Q and K
 *                rotated with the same signs, or both unrotated; V never
 *                rotated).
 *   q_descale, k_descale, v_descale : [B][H][ceil(N/128)] fp32 factors.
 *   o   : [B][H][N][d] bf16, written.   lse : [B][H][N] fp32 or NULL.
 *   d   : 64, 128 or 256 (others -> ATTN_ERR_UNSUPPORTED).
 *   v_transpose : 0 = feed V to the tensor core MN-major, straight from the
 *                 TMA tile; 1 = transpose each V tile in shared memory to
 *                 K-major first (the pages' layout step; sm_100a accepts
 *                 either, both give identical results).  1 needs d = 128
 *                 (ATTN_ERR_UNSUPPORTED at d = 64 and 256).
 * Scores use scale * q_descale * k_descale per (query block, key block);
 * P is rounded to e4m3 after multiplying by 256 * v_descale[j] / max_j
 * v_descale[j]; statistics are fp32 and l sums the unrounded P.
 */
attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                           const float* q_descale, const float* k_descale,
                           const float* v_descale, void* o, float* lse, int B, int H, int N,
                           int d, float scale, int causal, int v_transpose, void* stream);

/*
 * attn_last_status -- synchronises `stream`, then reads and clears the
 * current device's status word.  Returns ATTN_OK, ATTN_ERR_BOUNDS (debug build:
 * a range check failed), ATTN_ERR_TIMEOUT (a kernel
 * wait ran out; the affected outputs are undefined) or ATTN_ERR_CUDA.
 * `where` (may be NULL) receives 2 ints: the barrier id and block index
 * recorded with the error.
 */
attn_status_t attn_last_status(void* stream, int* where);

/*
 * attn_fwd_noalloc -- attn_fwd for callers that cannot allocate device
 * memory.  The pages have no counterpart: it exists for callers such as a
 * process whose device memory is owned by a pool allocator or another
 * runtime, or code that must not trigger cudaMalloc (whose first-use
 * allocation attn_fwd performs for its status word) at a point where
 * allocation is forbidden.
 *   Arguments, layout, validation, results and error codes are those of
 *   attn_fwd, except that only d == 64 and d == 128 are accepted: every
 *   other head dim (including 256 and the zero-padded sizes attn_fwd takes)
 *   returns ATTN_ERR_UNSUPPORTED.  Outputs are bit-identical to attn_fwd's
 *   for the same arguments (the same kernel and schedule run).
 *   The only scratch the kernel needs -- the 16-byte record its bounded
 *   waits write on a timeout -- lives in a static 256-byte device array
 *   inside the library instead of memory the library allocates.  That need
 *   does not grow with B, H, N or d, so no size exceeds the 256-byte
 *   maximum; every GPU that loads the library holds the array until exit.
 *   This entry point calls no cudaMalloc, cudaFree or allocating routine.
 *   Its first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   Every call clears the record on `stream` before its launch.  All calls
 *   share the one array, so calls whose kernels overlap on the GPU (on
 *   different streams) race on it.  A wait that runs out is recorded in that
 *   shared record, not in attn_fwd's status word: read it with
 *   attn_noalloc_last_status(); the outputs of a call that timed out are
 *   undefined.
 */
attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int N, int d, float scale, int causal, int dtype,
                               void* stream);

/*
 * attn_noalloc_last_status -- attn_last_status for attn_fwd_noalloc:
 * synchronises `stream`, then reads and clears the shared record of the
 * current device (through a host copy; nothing is allocated).  Returns
 * ATTN_OK or ATTN_ERR_TIMEOUT (a wait of the last noalloc launch ran out;
 * its outputs are undefined), ATTN_ERR_CUDA on a CUDA error.  `where` (may
 * be NULL) receives 2 ints: the barrier id and block index recorded with the
 * error.  With noalloc calls in flight on several streams the record holds
 * whichever error was written first since the last clear.
 */
attn_status_t attn_noalloc_last_status(void* stream, int* where);

/*
 * attn_bwd_workspace_bytes -- size of the workspace attn_bwd needs for these
 * sizes and mode: B * H * ceil(N / 128) * 256 * 4 bytes of row statistics
 * (two fp32 values per query row, rows padded to whole 128-row tiles), plus,
 * when `deterministic` is 0, B * H * N * d * 4 bytes of fp32 dQ accumulator.
 * Returns 0 for sizes < 1 or a mode other than 0 / 1.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int N, int d, int deterministic);

/*
 * attn_bwd -- 16-bit attention backward: the gradients of O with respect to
 * Q, K and V, given dO.  The chain rule of the definition above, with the
 * probabilities recomputed from the forward pass's LSE (P is never stored):
 *
 *   P  = exp(scale * Q K^T - LSE)   (0 where causal masking hides a key)
 *   dV = P^T dO
 *   dP = dO V^T,   D = rowsum(dO * O),   dS = P * (dP - D)
 *   dQ = scale * dS K,   dK = scale * dS^T Q
 *
 * The pages benchmark this pass beside the forward (quantum-bit repost
 * "H100 utilisation 75% ... FlashAttention-3", attention benchmark) without
 * writing it out; these are the standard gradients of softmax attention.
 *   q, k, v, o, d_o : [B][H][N][d] bf16 or fp16 (per `dtype`), read only;
 *                     o and lse as returned by attn_fwd for the same q, k,
 *                     v, scale and causal.
 *   lse             : [B][H][N] fp32 (natural log), read only.
 *   dq, dk, dv      : [B][H][N][d] same dtype, written.
 *   workspace       : device memory of at least attn_bwd_workspace_bytes(B,
 *                     H, N, d, deterministic) bytes, 16-byte aligned, owned
 *                     by the caller; its contents on entry do not matter
 *                     and are overwritten.
 *   d               : a multiple of 8, at most 128 (64 and 128 natively,
 *                     others zero-padded); larger d returns
 *                     ATTN_ERR_UNSUPPORTED.
 *   deterministic   : 0 -- fused path (three kernels): one pass over the key
 *                     tiles computes dK, dV and dQ; dQ is summed over key
 *                     tiles by fp32 TMA reduce-adds (atomic in L2) into the
 *                     workspace, so its last bits may differ from run to run
 *                     (dK, dV do not).
 *                     1 -- two kernels (dQ, then dK/dV), no atomics, every
 *                     output bit-reproducible; recomputes S and dP, so it
 *                     does seven N x N x d products instead of five.
 *   B, H, N, scale, causal, dtype, stream: as for attn_fwd.
 * Rounding: scores, P, dP and accumulation are fp32; P and dS are rounded to
 * the input dtype before the products that use them; D is accumulated in
 * fp32 from the 16-bit dO and O; outputs are rounded to the input dtype.
 * The "Results are deterministic" convention above holds for
 * deterministic = 1 only.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace,
                       size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                       int deterministic, int dtype, void* stream);

/*
 * attn_fwd_splitkv -- 16-bit attention forward for Nq queries against Nk
 * keys, the keys divided into splits processed in parallel and merged
 * (the decode-phase parallelisation over the key/value length the pages
 * attribute to FlashDecoding: "FlashAttention-3" explainer, droidorbit.com,
 * FAQ "How does FlashAttention-3 compare to FlashDecoding?").  Each split s
 * computes over its keys J_s the partial result O_s and LSE_s of the
 * definition above; the merge is the online-softmax rescaling across splits:
 * LSE = ln sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
 *   q, o    : [B][H][Nq][d] bf16 or fp16 (per `dtype`); o written.
 *   k, v    : [B][H][Nk][d] same dtype, read only.
 *   lse     : [B][H][Nq] fp32 (natural log), written; may be NULL.
 *   Nq, Nk  : >= 1, B*H*Nq and B*H*Nk < 2^31.
 *   causal  : 0 or 1.  Query i stands at position Nk - Nq + i: it sees keys
 *             j <= Nk - Nq + i (requires Nq <= Nk; with Nq = Nk this is
 *             attn_fwd's mask).
 *   n_splits: number of key splits per (batch, head, 128-query tile); 0
 *             picks one from the sizes and the SM count
 *             (attn_fwd_splitkv_auto_splits); larger than ceil(Nk / 128) is
 *             clamped to it.  Causal query tiles that see fewer key tiles use
 *             fewer splits.
 *   workspace: device memory of at least attn_fwd_splitkv_workspace_bytes(B,
 *             H, Nq, d, n_splits) bytes (with the split count actually used),
 *             16-byte aligned, owned by the caller, contents irrelevant:
 *             fp32 partial O_s [n_splits][B*H][Nq][d] then LSE_s.
 *   d       : a multiple of 8, at most 256 (64, 128 and 256 natively, others
 *             zero-padded to the next of those).
 *   scale, dtype, stream: as for attn_fwd.
 * Two kernels on `stream` (splits, then the merge).  Rounding: each split as
 * attn_fwd (fp32 statistics, P rounded to the input dtype) with O_s kept in
 * fp32; the merge is fp32; O is rounded once to the input dtype.
 */
attn_status_t attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int Nq, int Nk, int d, float scale, int causal,
                               int n_splits, int dtype, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Bytes of workspace attn_fwd_splitkv needs for `n_splits` splits (0 for
 * sizes < 1). */
size_t attn_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int d, int n_splits);

/* The split count attn_fwd_splitkv uses when given n_splits = 0, for the
 * current device (0 for sizes < 1 or a CUDA error). */
int attn_fwd_splitkv_auto_splits(int B, int H, int Nq, int Nk);

/*
 * attn_fwd_host -- attn_fwd on HOST buffers, the transfers overlapped with
 * the computation: the B*H heads are processed in chunks (about a
 * sixteenth of the heads each) through two device slots in `workspace`; the
 * host-to-device copies of chunk c+1 (one internal stream) and the
 * device-to-host copies of chunk c-1 (another) run while chunk c computes on
 * `stream`.  One cudaMemcpyAsync per tensor and chunk.
 *   q_host, k_host, v_host : [B][H][N][d] bf16 / fp16 in host memory (pinned
 *             memory for the copies to overlap; pageable memory works but
 *             its copies do not overlap).
 *   o_host  : [B][H][N][d] same dtype, host memory, written.
 *   lse_host: [B][H][N] fp32 host memory, written; may be NULL.
 *   workspace: device memory of at least attn_fwd_host_workspace_bytes(B, H,
 *             N, d) bytes, 16-byte aligned, owned by the caller.
 *   B, H, N, d, scale, causal, dtype: as for attn_fwd.
 * Asynchronous like attn_fwd: the call returns once everything is enqueued;
 * the results are in host memory when `stream` has completed (synchronize
 * it before reading o_host / lse_host).  The copies start after the work
 * already queued on `stream`.  The library keeps two internal streams and
 * seven events per device (created on first use, kept until exit); calls on
 * one device from several host threads take turns while they enqueue, and
 * their copies share the two internal streams.  Outputs are bit-identical
 * to attn_fwd on the same inputs.
 */
attn_status_t attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                            float* lse_host, int B, int H, int N, int d, float scale, int causal, int dtype,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace attn_fwd_host needs (0 for sizes < 1). */
size_t attn_fwd_host_workspace_bytes(int B, int H, int N, int d);

/* Static description of a status code. */
const char* attn_status_string(attn_status_t s);

/*
 * attn_debug_set_fault -- test hook for the bounded waits.  When `mode` is 1
 * the next attn_fwd launch runs with its TMA producer told to skip its first
 * load-complete arrival, so the consumers' waits must run out: the call
 * returns ATTN_OK and attn_last_status() then reports ATTN_ERR_TIMEOUT.  The
 * hook resets itself after one launch.  `wait_limit_ms` (> 0) overrides the
 * wait limit for that launch.  No device fault, trap or hang is involved.
 * Mode 2 exists in the debug build only (ATTN_ERR_UNSUPPORTED otherwise): the
 * next attn_fwd launch checks CTA 0's first S load of TMEM as if its columns
 * were out of range, so attn_last_status() reports ATTN_ERR_BOUNDS (where =
 * the check's id, 29); the load itself is never out of range: the failed check
 * skips it, and that launch's outputs are undefined.
 */
attn_status_t attn_debug_set_fault(int mode, int wait_limit_ms);

/*
 * attn_debug_set_ablation -- bench hook for the pages' ablation of the
 * overlap between the softmax and the matmuls (quantum-bit repost "H100
 * utilisation 75% ... FlashAttention-3", ablation paragraph).  While `mode`
 * is 1, attn_fwd / attn_fwd_strided / attn_fwd_host calls with bf16 inputs
 * and head dim 128 (native, not padded) run a variant of the kernel whose two
 * query tiles are serialised: the tensor core waits until both tiles have
 * turned S into P before any product of the next key tile, and both tiles'
 * next S are published together, so no product overlaps a softmax.  Results
 * are bit-identical to mode 0 (the same products and roundings in the same
 * order); only the schedule differs.  Other dtypes and head dims return
 * ATTN_ERR_UNSUPPORTED while the mode is 1; attn_fwd_noalloc and
 * attn_fwd_fp8 ignore it.  Mode 0 (the default) restores the ping-pong
 * schedule.  The setting is global to the process and stays until changed.
 * Returns ATTN_ERR_INVALID_ARG for other modes.
 */
attn_status_t attn_debug_set_ablation(int mode);

/*
 * attn_debug_status_allocated -- test query: 1 if the current device's
 * attn_fwd status word (the one allocation the library makes on first use of
 * a device) exists, 0 if not, -1 on a CUDA error.  Lets a test check that
 * attn_fwd_noalloc and attn_noalloc_last_status allocate nothing.
 */
int attn_debug_status_allocated(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_SM100_H_ */
