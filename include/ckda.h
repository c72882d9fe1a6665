/*
 * ckda.h -- C ABI of the B200 (sm_100a) Complex KDA (CKDA) recurrence library.
 *
 * The recurrence (per batch b and head h, sequential over tokens t):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   S in R^{dk x dv}
 *     o_t = scale * S_t^T q_t,                                                 scale = dk^-1/2
 *
 * with a signed channel-wise gate alpha_t in [-1, 1]^dk and beta_t in [0, 2].  The transition
 * (I - beta k k^T) Diag(alpha) is the gated delta-rule transition of the "Complex KDA" paper
 * summary (picx.dev), "Background"; the ranges are its "CKDA Definition".  Before the recurrence
 * q_t and k_t are optionally rotated (rotary embedding at position pos_offset + t, inverse
 * frequencies rope_theta^(-2i/dk), "RoPE into the KDA q/k path" review, section 5) and then
 * L2-normalised per head, x / sqrt(sum x^2 + 1e-6) (the same review, sections 2-3: the norm is
 * a kernel-side step and the rotation comes before it).
 *
 * Conventions shared by every entry point:
 *  - Every array pointer is CALLER-OWNED DEVICE memory (cudaMalloc / torch) on the current
 *    device.  The library never allocates, frees or retains memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *    A returned CKDA_OK means the arguments were valid and the kernels were enqueued; kernel
 *    execution errors surface at the next synchronisation, as with any CUDA launch.
 *  - Arguments are validated on the host before anything is launched; on any error nothing is
 *    launched and no output is touched.  Values are not inspected: NaN/Inf propagate, and
 *    alpha outside [-1, 1] or beta outside [0, 2] are accepted as given.
 *  - Array pointers must be 16-byte aligned.  Outputs must not overlap inputs (except the
 *    decode state, which is updated in place by design).
 *  - Layouts are dense row-major with the last index fastest:
 *        q, k, alpha : [B, T, H, dk]     v, out : [B, T, H, dv]     beta : [B, T, H]
 *        h0, hT, decode state : [B or N, H, dk, dv]  (fp32 always)
 *    q, k, v, out have the element type `dtype`; beta and states are fp32; alpha is fp32 gate
 *    values, or (flags.gate_logits = 1) logits of the element type `dtype`.
 *  - Supported sizes: dk, dv in {16, 32, 64, 128}; chunk in {16, 32, 64}; any T >= 1 (a
 *    partial last chunk is handled exactly).  B*H, N*H >= 1.
 *  - Failures the kernels detect on the device (a bounded wait of the tensor-core forward that
 *    ran out, packed-sequence offsets whose device copy disagrees with the host copy) are
 *    recorded in a per-device status word instead of faulting: the kernel stops its work, leaves
 *    the outputs unspecified and returns, so the context stays usable.  The call itself has
 *    already returned CKDA_OK by then; ckda_last_device_status reports the failure.
 */
#ifndef CKDA_H
#define CKDA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CKDA_ABI_VERSION 7

#if defined(__GNUC__)
#define CKDA_API __attribute__((visibility("default")))
#else
#define CKDA_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* ckda_stream_t;

typedef enum {
    CKDA_OK = 0,
    CKDA_ERR_NULL = 1,        /* a required pointer is NULL */
    CKDA_ERR_SHAPE = 2,       /* a size is out of range (T < 1, B*H < 1, overflow, ...) */
    CKDA_ERR_UNSUPPORTED = 3, /* dk, dv, chunk, dtype or path outside the compiled set */
    CKDA_ERR_ALIGN = 4,       /* an array pointer is not 16-byte aligned */
    CKDA_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than ckda_fwd_workspace_bytes() */
    CKDA_ERR_CUDA = 6,        /* a CUDA runtime call failed while configuring or launching */
    CKDA_ERR_ARG = 7,         /* any other invalid argument (flags, overlapping buffers) */
    CKDA_ERR_DEVICE_STATUS = 8 /* a kernel recorded a failure in the device status word
                                  (ckda_last_device_status) */
} ckda_status;

typedef enum {
    CKDA_F32 = 0,  /* q, k, v, out are float32 */
    CKDA_BF16 = 1  /* q, k, v, out are bfloat16; all arithmetic accumulates in fp32 */
} ckda_dtype;

typedef enum {
    CKDA_PATH_AUTO = 0,  /* tensor-core path where compiled (bf16, dk = dv = 128, chunk = 64) */
    CKDA_PATH_SIMT = 1,  /* fp32 CUDA-core chunked path, every supported size and dtype */
    CKDA_PATH_TC = 2     /* tensor-core path (tcgen05); CKDA_ERR_UNSUPPORTED elsewhere */
} ckda_path;

typedef struct {
    int l2norm;          /* nonzero: L2-normalise q and k per head, after the rotation */
    float rope_theta;    /* > 0: rotary base (10000 is the usual); <= 0: no rotation */
    int rope_convention; /* 0: half-split pairs (x_i, x_{i+dk/2}); 1: interleaved (x_{2i}, x_{2i+1}) */
    float scale;         /* read-out scale; 0 selects dk^-1/2 */
    int path;            /* ckda_path; ckda_fwd_chunked only, ignored elsewhere */
    int stages;          /* ckda_fwd_chunked on the tensor-core path only: 0 = one fused
                            launch (chunk-parallel factor work and the serial state pass run
                            side by side); profiling aids: 3 = the two parts as two kernels in
                            sequence, 1 = only the factor kernel (fills the workspace), 2 = only
                            the state pass (reads a workspace filled by a stage-1 call with the
                            same arguments) */
    int gate_logits;     /* 0: alpha and beta hold the gates themselves (fp32).  1: they hold
                            logits -- alpha the logits a in the element type `dtype`, beta the
                            logits b in fp32 -- and the kernels form the gates as
                            alpha = 2 sigma(a) - 1 and beta = 2 sigma(b), sigma the logistic
                            function (the parameterisation of the "Complex KDA" paper summary,
                            Methodology, CKDA Definition).  Any other value: CKDA_ERR_ARG. */
    int rope_dims;       /* channels rotated when rope_theta > 0: 0 or dk = all; dk / 2 (dk >= 32)
                            = the first half of each head's channels, as a rotation of that
                            sub-vector on its own (pairs and frequencies theta^(-2i/(dk/2)) over
                            those channels; the "RoPE review", section 3, partial rotation); the
                            other channels are carried through, and the L2 norm, after it, covers
                            all dk.  Other values: CKDA_ERR_ARG. */
    int qk_heads;        /* grouped value heads (GVA): 0 = q and k have the same H heads as v;
                            otherwise q and k have qk_heads heads (which must divide H) and value
                            head h reads q and k head h / (H / qk_heads), i.e. each q/k head is
                            repeated H / qk_heads times on the head axis.  The rotation and the
                            L2 norm act on q and k before the repeat ("RoPE review", section 7,
                            on the GVA repeat).  alpha, beta, v, out and the states stay on the H
                            value heads.  Negative, or not dividing H: CKDA_ERR_ARG.
                            ckda_fwd_chunked, ckda_fwd_varlen and ckda_decode_step; ignored
                            elsewhere. */
} ckda_flags;

/* Version of this ABI (CKDA_ABI_VERSION of the build). */
CKDA_API int ckda_abi_version(void);

/* Human-readable text for a status code (static storage, never NULL). */
CKDA_API const char* ckda_strerror(ckda_status status);

/*
 * Device status word of the current device: waits until `stream` has finished its work, then
 * reads the word and clears it.  The word is shared by every stream and call on the device and
 * keeps the first failure recorded since the last read.  *code (may be NULL) receives it:
 *   0  no failure recorded
 *   1  a wait of the tensor-core forward's chunk-factor work ran out (a poll limit)
 *   2  a wait of the tensor-core forward's state pass ran out (ckda_set_wait_limit_ns)
 *   3  ckda_fwd_varlen: the device copy of cu_seqlens disagrees with the host copy
 * Returns CKDA_OK for 0, CKDA_ERR_DEVICE_STATUS otherwise, CKDA_ERR_CUDA when the read fails.
 * After a recorded failure the outputs of the failing call are unspecified.  There is no
 * counterpart on the pages: it reports the bounded waits of this library's own kernels.
 */
CKDA_API ckda_status ckda_last_device_status(ckda_stream_t stream, int* code);

/*
 * Upper bound, in nanoseconds, of any single wait of the tensor-core forward's state pass on the
 * current device (a wait for a chunk's factors to be produced, or for a tensor-core product).
 * A wait that reaches it stops the kernel with status 2.  ns = 0 restores the default, 4 s,
 * which no correct run comes near (the state pass waits at most for one head group's factors).
 * Synchronous; affects calls enqueued afterwards.  A diagnostic, with no counterpart on the
 * pages: a short limit lets a test make a wait run out on purpose.
 */
CKDA_API ckda_status ckda_set_wait_limit_ns(unsigned long long ns);

/*
 * Prologue alone: q_out = L2(rope(q)), k_out = L2(rope(k)) per head, with the rotation at
 * position pos_offset + t.  q, k, q_out, k_out: [B, T, H, dk] of `dtype` (arithmetic in fp32).
 * The rotary embedding and the placement of the norm after it follow the "RoPE into the KDA
 * q/k path" review, sections 2, 3 and 5.  In-place use (q_out == q, k_out == k) is allowed.
 * dk in {16, 32, 64, 128}.
 */
CKDA_API ckda_status ckda_qk_prologue(const void* q, const void* k, void* q_out, void* k_out, int B, int T,
                             int H, int dk, ckda_flags flags, ckda_dtype dtype,
                             long long pos_offset, ckda_stream_t stream);

/*
 * Bytes of device workspace ckda_fwd_chunked needs for this problem and path selection
 * (`path` as in ckda_flags).  Returns 0 when no workspace is needed, and (size_t)-1 when the
 * sizes are invalid or unsupported for that path.
 */
CKDA_API size_t ckda_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk, ckda_dtype dtype,
                                int path);

/*
 * Chunked forward over whole sequences.
 *   q, k   : [B, T, Hk, dk] dtype         v   : [B, T, H, dv] dtype
 *            (Hk = flags.qk_heads, or H when that is 0)
 *   alpha  : [B, T, H, dk] fp32 gates (signed), or dtype logits when flags.gate_logits
 *   beta   : [B, T, H] fp32 gates, or fp32 logits when flags.gate_logits
 *   h0     : [B, H, dk, dv] fp32, or NULL for a zero initial state
 *   out    : [B, T, H, dv] dtype (written)
 *   hT     : [B, H, dk, dv] fp32 final state, or NULL to skip it (may equal h0: read before write
 *            is guaranteed per (b, h))
 *   chunk  : tokens per chunk of the chunked evaluation (16, 32 or 64; the tensor-core path
 *            needs 64); the result does not depend on it beyond rounding.
 *   pos_offset : rotary position of token t is pos_offset + t (used when rope_theta > 0).
 *   workspace / workspace_bytes : device scratch of at least ckda_fwd_workspace_bytes(...),
 *            16-byte aligned; may be NULL when that is 0.  Owned by the caller; it must not be
 *            shared by calls that can run concurrently.
 * The computation is the recurrence above, evaluated chunk by chunk: within a chunk a WY/UT
 * representation of the product of transitions, across chunks an fp32 state.
 */
CKDA_API ckda_status ckda_fwd_chunked(const void* q, const void* k, const void* v, const void* alpha,
                             const float* beta, const float* h0, void* out, float* hT, int B,
                             int T, int H, int dk, int dv, int chunk, ckda_flags flags,
                             ckda_dtype dtype, long long pos_offset, void* workspace,
                             size_t workspace_bytes, ckda_stream_t stream);

/*
 * Bytes of the optional workspace of the CUDA-core path (flags.path = CKDA_PATH_SIMT, or sizes
 * the tensor-core path does not take), or (size_t)-1 for invalid sizes.  Given to
 * ckda_fwd_chunked as its workspace (at least this many bytes, 16-byte aligned), it selects the
 * record form of that path: every 16-token chunk's factors formed once, chunk-parallel, and the
 * serial pass over the chunks with the products on warp-level tensor-core tiles (split tf32
 * operands, fp32-grade); without it (and for packed sequences) the path recomputes the chunk
 * factors in plain fp32 loops per 16 state columns.  Both give the recurrence up to rounding.
 * ckda_fwd_workspace_bytes reports 0 for this path (the workspace is not required).
 */
CKDA_API size_t ckda_fwd_simt_workspace_bytes(int B, int T, int H, int dk, int dv);

/*
 * The chunked forward with a segment-parallel state pass (tensor-core path only: bf16,
 * dk = dv = 128, chunk 64; batched sequences).  The serial pass over the chunks of every
 * (batch, head) is split into `segments` segments of L = ceil(ceil(T/64) / segments) chunks
 * (as many as that needs, none empty).  Every chunk's transition is
 *     A_c = Diag(gamma_C) - K_end^T W      (dk x dk),
 * the chunk-level form of the product of the per-token transitions (I - beta k k^T) Diag(alpha)
 * of the "Complex KDA" paper summary, "Background"; the summary's fixed-size state is what makes
 * a segment's composition F_s = A_c(last) ... A_c(first) a dk x dk matrix.  A summary pass forms,
 * in parallel over segments, each segment's end state from zero (from h0 for the first) and its
 * transition F_s; an fp32 scan forms the state entering every segment, S_{s+1} = F_s S_s + E_s;
 * a second parallel pass runs every segment from its entering state and writes the outputs
 * (and hT).  The result is the recurrence's, like ckda_fwd_chunked's, up to rounding; the work
 * on the serial path drops from ceil(T/64) chunk steps to about 3 L + segments, for about three
 * times the state-pass products in total.  It pays when few (batch, head) pairs carry long
 * sequences (ckda_fwd_segments_auto).
 *   Arguments as ckda_fwd_chunked (chunk fixed at 64; flags.path must not select the CUDA-core
 *   path, flags.stages is ignored), plus
 *   segments : >= 1; 1 runs ckda_fwd_chunked's single fused launch.
 *   workspace / workspace_bytes : at least ckda_fwd_segmented_workspace_bytes(...): the
 *            tensor-core forward's workspace and three fp32 arrays of B*H*P dk x dv matrices.
 * Errors: CKDA_ERR_UNSUPPORTED outside the tensor-core sizes (segments > 1), CKDA_ERR_ARG for
 * segments < 1, otherwise as ckda_fwd_chunked.  hT may equal h0 (h0 is read by the first two
 * launches, hT written by the last).
 */
CKDA_API size_t ckda_fwd_segmented_workspace_bytes(int B, int T, int H, int dk, int dv,
                                                   int segments);
CKDA_API ckda_status ckda_fwd_segmented(const void* q, const void* k, const void* v,
                                        const void* alpha, const float* beta, const float* h0,
                                        void* out, float* hT, int B, int T, int H, int dk,
                                        int dv, ckda_flags flags, ckda_dtype dtype,
                                        long long pos_offset, int segments, void* workspace,
                                        size_t workspace_bytes, ckda_stream_t stream);
/*
 * Segment count for ckda_fwd_segmented on the current device from a cycle model of the four
 * launches against the single fused launch; 1 when the fused launch is expected to be faster
 * (many (batch, head) pairs keep every SM busy with chunk-parallel work).
 */
CKDA_API int ckda_fwd_segments_auto(int B, int T, int H);

/*
 * Bytes of device workspace ckda_fwd_varlen needs for these packed sequences (cu_seqlens_host as
 * below) and path selection.  0 when none is needed; (size_t)-1 when the offsets or sizes are
 * invalid or unsupported for that path.
 */
CKDA_API size_t ckda_fwd_varlen_workspace_bytes(const int* cu_seqlens_host, int n_seqs, int H,
                                                int dk, int dv, int chunk, ckda_dtype dtype,
                                                int path);

/*
 * Chunked forward over packed sequences of different lengths: n_seqs sequences laid end to end
 * on one token axis of T_total = cu_seqlens_host[n_seqs] tokens, described by token offsets
 * (the cu_seqlens layout with which FLA's attention layer rotates packed sequences: "RoPE into
 * the KDA q/k path" review, section 4).  Sequence s owns tokens cu[s] .. cu[s+1] - 1; it starts
 * from h0[s] (or zero), ends in hT[s], and the rotary position of its token t (t counted from
 * its first token) is pos_offset + t.  No state passes from one sequence to the next: the
 * result for each sequence is the ckda_fwd_chunked result for that sequence alone.
 *   q, k   : [T_total, Hk, dk] dtype       v, out : [T_total, H, dv] dtype
 *   alpha  : [T_total, H, dk], beta : [T_total, H]  (values or logits as flags.gate_logits)
 *   h0, hT : [n_seqs, H, dk, dv] fp32 (h0 may be NULL, hT may be NULL or equal h0)
 *   cu_seqlens      : device int32 [n_seqs + 1], 4-byte aligned, read by the kernels
 *   cu_seqlens_host : host int32 [n_seqs + 1], the same values, read before the call returns
 *                     (it sizes the launch): cu[0] = 0 and non-decreasing, else CKDA_ERR_ARG.
 *                     Empty sequences are allowed (their hT is h0, or zero).  If the two copies
 *                     differ, the results are undefined, but every access stays inside the
 *                     arrays described by cu_seqlens_host.
 *   n_seqs >= 1; the other arguments as ckda_fwd_chunked, with workspace of at least
 *   ckda_fwd_varlen_workspace_bytes(...).
 * On the tensor-core path each head's chain of chunk steps runs through the sequences in turn;
 * a sequence's last chunk may be short (its own tokens only are written).
 */
CKDA_API ckda_status ckda_fwd_varlen(const void* q, const void* k, const void* v,
                                     const void* alpha, const float* beta, const float* h0,
                                     void* out, float* hT, const int* cu_seqlens,
                                     const int* cu_seqlens_host, int n_seqs, int H, int dk, int dv,
                                     int chunk, ckda_flags flags, ckda_dtype dtype,
                                     long long pos_offset, void* workspace,
                                     size_t workspace_bytes, ckda_stream_t stream);

/*
 * One decode step for N independent sequences, in place on the caller's fp32 state:
 *   q, k : [N, Hk, dk] (Hk = flags.qk_heads, or H)    alpha : [N, H, dk]
 *   v, out : [N, H, dv]    beta : [N, H]
 *   (alpha fp32 gates or dtype logits, beta fp32 gates or logits, as flags.gate_logits says)
 *   state       : [N, H, dk, dv] fp32, read and overwritten with S_t
 *   pos         : [N] int64 rotary positions (required when rope_theta > 0, else ignored)
 * out = scale * S_t^T q_t, with S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T.
 * Each head's state is streamed through the SM exactly once (read once, written once).
 */
CKDA_API ckda_status ckda_decode_step(const void* q, const void* k, const void* v, const void* alpha,
                             const float* beta, float* state, void* out, const long long* pos,
                             int N, int H, int dk, int dv, ckda_flags flags, ckda_dtype dtype,
                             ckda_stream_t stream);

/*
 * Bytes of device workspace ckda_bwd_chunked needs (never 0), or (size_t)-1 for invalid or
 * unsupported sizes.
 */
CKDA_API size_t ckda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);

/*
 * Backward of ckda_fwd_chunked: the gradients of L = <dout, out> + <dhT, hT> with respect to
 * q, k, v, the gates and h0, for the forward with the same inputs, sizes and flags (rotation,
 * norm, scale, grouped value heads, gate logits).  Computed in fp32-grade arithmetic (fp32 on
 * the CUDA cores; the dense products as warp-level tensor-core tiles whose tf32 operands are split
 * into a head and a remainder, about 3 * 2^-20 relative per product) by the chunked form
 * run in reverse (16-token chunks: the forward replay keeps each chunk's entering
 * state, a reverse chain carries the state gradient, every chunk forms its input gradients, and
 * the prologue -- rotation, then L2 norm -- is differentiated last).  There is no backward on
 * the pages beyond the statement that one exists ("Complex KDA" paper summary, Implementation:
 * a hybrid TileLang backward); this is the reverse mode of the recurrence above.
 *   q, k, v, alpha, beta, h0 : the forward's inputs (layouts and types as ckda_fwd_chunked;
 *                              h0 may be NULL for a zero initial state)
 *   dout : [B, T, H, dv] of `dtype`, the gradient of out (required)
 *   dhT  : [B, H, dk, dv] fp32, the gradient of hT, or NULL for zero
 *   dq, dk : [B, T, Hk, dk] fp32 (Hk = flags.qk_heads or H: a grouped q/k head receives the sum
 *            over the value heads that read it)
 *   dv   : [B, T, H, dv] fp32      dalpha : [B, T, H, dk] fp32      dbeta : [B, T, H] fp32
 *          (with flags.gate_logits, dalpha and dbeta are the gradients of the logits a and b)
 *   dh0  : [B, H, dk, dv] fp32, or NULL to skip it
 *   workspace : at least ckda_bwd_workspace_bytes(B, T, H, dk, dv), 16-byte aligned, owned by
 *               the caller and not shared with concurrent calls
 * flags.path and flags.stages are ignored.  Outputs must not overlap the inputs or each other.
 */
CKDA_API ckda_status ckda_bwd_chunked(const void* q, const void* k, const void* v,
                                      const void* alpha, const float* beta, const float* h0,
                                      const void* dout, const float* dhT, float* dq, float* dk,
                                      float* dv, float* dalpha, float* dbeta, float* dh0, int B,
                                      int T, int H, int dk_, int dv_, ckda_flags flags,
                                      ckda_dtype dtype, long long pos_offset, void* workspace,
                                      size_t workspace_bytes, ckda_stream_t stream);

/*
 * Diagnostic: D[M, N] (fp32, row-major) = A[M, K] * B for bf16 A (row-major, K contiguous),
 * computed by the library's own tcgen05 tensor-core wrappers (shared-memory operand
 * descriptors with the 128-byte swizzle, TMEM accumulator, one CTA).
 *   b_mn_major bit 0 clear: B is [N, K] row-major (K contiguous), D = A B^T  (K-major B operand)
 *   b_mn_major bit 0 set:   B is [K, N] row-major (N contiguous), D = A B    (MN-major B operand)
 *   b_mn_major bit 1 set:   A is staged from shared memory into Tensor Memory with
 *                           tcgen05.cp and read by the product from there (M = 128 only)
 *   b_mn_major bit 2 set:   A is written into Tensor Memory by the threads with tcgen05.st
 *                           (row m in lane m, K elements 2j and 2j + 1 packed in column j) and
 *                           read by the product from there (M = 128 only)
 *   bits 1 and 2 together, or other bits: CKDA_ERR_ARG.
 * M in {64, 128}; N a multiple of 16 in [16, 256] (32 or a multiple of 64 when b_mn_major);
 * K a multiple of 64 in [64, 256].  Lets a user check the tensor-core path on a device.
 */
CKDA_API ckda_status ckda_selftest_umma(const void* A, const void* B, float* D, int M, int N, int K,
                               int b_mn_major, ckda_stream_t stream);

/*
 * ckda_fwd_chunked without a caller-supplied workspace (the paper has no counterpart; this is a
 * deployment convenience).  For callers that cannot allocate device memory where they run the
 * forward -- inside CUDA-graph stream capture, under a fixed start-up memory pool, or on a
 * real-time path that must not call cudaMalloc/cudaFree -- the scratch lives in a fixed device
 * array of CKDA_NOALLOC_MAX_WORKSPACE bytes inside the library, held by every GPU that loads it
 * until the process exits.  The function allocates nothing.
 *   Arguments and results: as ckda_fwd_chunked, minus workspace / workspace_bytes.
 *   Limit: problems whose ckda_fwd_workspace_bytes(...) exceeds CKDA_NOALLOC_MAX_WORKSPACE are
 *          rejected with CKDA_ERR_WORKSPACE before anything is launched (16 MiB holds 186
 *          chunk-heads of the tensor-core path: B * H * ceil(T / 64) <= 186).
 *   Set-up: the first call on a device looks up the array's device address (cudaGetSymbolAddress,
 *          with that device current); make that first call before any stream capture.
 *   Sharing: every call uses the same array, which keeps the last call's contents (no part of it
 *          needs to start at zero).  Calls whose work overlaps on the GPU race on it: issue them
 *          on one stream, or otherwise order them.
 *   flags.stages: 0 or 3 only (each of those clears the array's ready flags itself); the
 *          profiling stages 1 and 2 are refused with CKDA_ERR_ARG, since a stage-2 call would
 *          read whatever an earlier call, of any shape, left in the shared array.
 */
#define CKDA_NOALLOC_MAX_WORKSPACE (16u << 20)

CKDA_API ckda_status ckda_fwd_chunked_noalloc(const void* q, const void* k, const void* v,
                                              const void* alpha, const float* beta,
                                              const float* h0, void* out, float* hT, int B,
                                              int T, int H, int dk, int dv, int chunk,
                                              ckda_flags flags, ckda_dtype dtype,
                                              long long pos_offset, ckda_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CKDA_H */
