/*
 * gdr.h -- C ABI of the gated delta-rule sequence mixer for NVIDIA B200
 * (sm_100a).
 *
 * The mixer keeps a matrix state S (d_v x d_k, row i = value channel,
 * column j = key channel) and, for every token t,
 *
 *     S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * Sources:
 *   "Decoding Hybrid Linear Attention Architectures", section 3 (state
 *   update equations: item 3 Gated Delta Rule with a scalar gate, item 6
 *   Gated Delta Attention with a per-channel gate and the decay -> erase ->
 *   write pseudocode), section 4 (the two gates), section 5 (chunkwise
 *   algorithm: inter-chunk state recursion, intra-chunk output, gates
 *   accumulated in log space) and section 6 (constant-cost decode step);
 *   "Linear Attention Variants (RetNet, GLA, DeltaNet, Based)", section
 *   "DeltaNet: Error-Correcting Writes" (the delta rule and its WY-based
 *   chunked parallel form).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer is a CUDA device pointer owned by the caller.  The library
 *   allocates no device memory in any call and keeps no per-call state.
 * - All device work is enqueued on `stream` (a cudaStream_t; NULL means the
 *   legacy default stream) and runs asynchronously.
 * - Argument errors are detected on the host, before anything is enqueued:
 *   the call returns GDR_ERR_INVALID_ARG or GDR_ERR_UNSUPPORTED and launches
 *   nothing; gdr_last_error_message() then describes the problem.
 * - A kernel that gives up a bounded wait records GDR_ERR_TIMEOUT in a
 *   device status word; gdr_get_device_status() reads and clears it.  The
 *   tensor-core path records GDR_ERR_RANGE there when a per-channel gate
 *   decays beyond what it can represent (see gdr_chunk_fwd).
 * - Gate: `g` holds log(alpha) in fp32 (finite, <= 0).  A scalar gate has one
 *   value per (token, head); a per-channel gate has d_k values.
 * - Dtypes: q, k, v and o share `in_dtype` (fp32 or bf16); g, beta and the
 *   state are always fp32.  All arithmetic accumulates in fp32.
 * - No query scale is applied: o_t = S_t q_t exactly as written above.
 * - Supported head sizes: d_k, d_v in {32, 64, 128}.  Chunk size C = 64.
 * - Pointers must be 16-byte aligned; every tensor is dense row-major
 *   (contiguous) in the layout given below.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDR_OK = 0,
  GDR_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad enum   */
  GDR_ERR_UNSUPPORTED = 2, /* valid request this build does not implement   */
  GDR_ERR_WORKSPACE = 3,   /* workspace pointer/size too small              */
  GDR_ERR_CUDA = 4,        /* a CUDA runtime call failed                    */
  GDR_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait (device word) */
  GDR_ERR_RANGE = 6        /* per-channel decay beyond the tensor-core path's
                              range in some chunk (device word)             */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

typedef enum { GDR_GATE_SCALAR = 0, GDR_GATE_PER_CHANNEL = 1 } gdr_gate_kind;

/* Same type as cudaStream_t. */
typedef struct CUstream_st *gdr_stream_t;

/*
 * Workspace the chunked forward needs for this problem on the current
 * device, in bytes (0 if none).  Pass at least this much (16-byte aligned,
 * device memory owned by the caller) to gdr_chunk_fwd.  Only long sequences
 * with few (b, h) use it: with B*H*P <= the device's SM count for a power of
 * two P >= 4 and T a multiple of 64*P with at least 16 chunks per segment,
 * each sequence runs as P segments (section 5 of "Decoding Hybrid Linear
 * Attention Architectures": a stretch's end state is its start state times
 * the stretch's transition plus what the stretch writes), which needs
 * 3 * B*P*H * dv*dk fp32 values of scratch.
 */
size_t gdr_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int C,
                                     gdr_dtype in_dtype, gdr_gate_kind gate);

/*
 * Number of kernels one gdr_chunk_fwd call with these arguments launches on
 * the current device (4 on the segment path, 1 otherwise, 0 if B*H == 0),
 * for sizing CUDA graphs and counting launches.
 */
int gdr_chunk_fwd_kernel_launches(int B, int T, int H, int dk, int dv, int C,
                                  gdr_dtype in_dtype, gdr_gate_kind gate);

/*
 * Chunkwise-parallel forward over whole sequences (prefill / training
 * forward).  Source: "Decoding Hybrid Linear Attention Architectures",
 * section 5; the per-token result it reproduces is the recurrence above.
 *
 *   q, k  [B, T, H, dk]  in_dtype      queries / keys (the caller normalises)
 *   v     [B, T, H, dv]  in_dtype      values
 *   g     [B, T, H]      fp32          log alpha, scalar gate, or
 *         [B, T, H, dk]  fp32          log alpha, per-channel gate
 *   beta  [B, T, H]      fp32          write strength in [0, 1]
 *   S0    [B, H, dv, dk] fp32 or NULL  initial state (NULL = zero state)
 *   o     [B, T, H, dv]  in_dtype      output (written)
 *   S_T   [B, H, dv, dk] fp32 or NULL  final state (written if not NULL)
 *   C     chunk length; must be 64
 *   workspace, ws_bytes: see gdr_chunk_fwd_workspace_bytes (may be NULL/0
 *         when that returns 0)
 *
 * T may be any value >= 0 (a ragged last chunk is masked); B*H may be 0.
 * S0 may alias S_T (each (b, h) reads all of S0 before writing S_T); o must
 * not alias any input.
 *
 * Two tensor-core kernels serve this call: bf16 with dk = dv = 128 runs the
 * warp-specialised kernel (bf16 operands); fp32 inputs and every other
 * (dk, dv) run the split-operand kernel, which carries each operand as two
 * bf16 terms and each product as three MMAs (close to fp32 accuracy).
 *
 * Range of per-channel gates: a chunk's K and Q tiles are scaled per key
 * channel by e^{+-(gc - m)} around the cumulative decay m at the chunk's
 * row 31, so in every channel the decay accumulated over each half chunk
 * (32 tokens) must stay above about -83 (bf16, dk = dv = 128; e.g. a decay
 * of e^{-2.6} per token held for 32 tokens) or -69 (split-operand kernel,
 * whose low terms must stay normal numbers).  A chunk beyond that has its
 * overflowing tile entries zeroed (the outputs stay finite but are not the
 * recurrence's) and the call records GDR_ERR_RANGE in the device status
 * word (gdr_get_device_status).  Scalar gates have no limit.
 */
gdr_status gdr_chunk_fwd(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                         const float *g, gdr_gate_kind gate, const float *beta,
                         const float *S0, void *o, float *S_T, int B, int T, int H, int dk,
                         int dv, int C, void *workspace, size_t ws_bytes,
                         gdr_stream_t stream);

/*
 * The chunked forward as P segments per sequence, with P chosen by the
 * caller, allocating nothing: every intermediate lives in the caller's
 * workspace.  Source: "Decoding Hybrid Linear Attention Architectures",
 * section 5, whose inter-chunk recursion (end state = start state times the
 * chunk's transition plus what the chunk writes) is applied per segment:
 * every segment runs from a zero state (the first from S0), giving E_p, and
 * from the identity with v taken as zero, giving its transition M_p; the
 * segments' start states follow in fp32 (S_start(p+1) = S_start(p) M_p +
 * E_p), and a last pass writes o.  gdr_chunk_fwd takes
 * this path by itself for long sequences with few heads; this entry point
 * fixes P (for example to capture a fixed shape in a CUDA graph).
 *
 * Arguments as gdr_chunk_fwd, plus
 *   P          segments per sequence, >= 2, T a multiple of 64*P
 *   workspace  device memory of at least 3*B*P*H*dv*dk*4 bytes, 16-byte
 *              aligned, owned by the caller (overwritten)
 * Needs bf16 inputs and dk = dv = 128 (GDR_ERR_UNSUPPORTED otherwise, also
 * for a P that does not split T into whole chunks); GDR_ERR_WORKSPACE if
 * the workspace is missing or too small.  Launches 4 kernels on `stream`.
 */
gdr_status gdr_chunk_fwd_segmented(const void *q, const void *k, const void *v,
                                   gdr_dtype in_dtype, const float *g, gdr_gate_kind gate,
                                   const float *beta, const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int dk, int dv, int C, int P,
                                   void *workspace, size_t ws_bytes, gdr_stream_t stream);

/* Size of the scratch array built into the library for
 * gdr_chunk_fwd_segmented_noalloc: 24 MiB, enough for B*P*H <= 128
 * segment-heads (for example one 65536-token sequence of 16 heads cut into
 * 8 segments). */
#define GDR_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)

/*
 * gdr_chunk_fwd_segmented without a workspace argument: the same segment
 * path and the same kernels, with the scratch taken from a fixed array that
 * is part of the library instead of from the caller.  It is meant for
 * callers that cannot allocate device memory when they run the mixer: a
 * plugin inside a host framework that owns the device's memory pool and
 * gives the plugin no allocator, or a serving loop that must not stall on
 * cudaMalloc / cudaFree, which can synchronise the whole device.  The
 * method on the pages has no counterpart of this entry point; the
 * arithmetic is that of gdr_chunk_fwd_segmented.
 *
 * Arguments as gdr_chunk_fwd_segmented without workspace / ws_bytes.  The
 * caller still owns and passes every input and output.
 *
 * Scratch: 3 * B*P*H * dv*dk * 4 bytes are needed; more than
 * GDR_NOALLOC_SCRATCH_BYTES is refused with GDR_ERR_WORKSPACE before
 * anything is enqueued.  The array is reserved on every GPU that loads the
 * library and held until the process exits.  Every call uses the same
 * array: two calls whose work overlaps on the GPU (on different streams, or
 * from different host threads) race on it and give undefined results, so
 * serialise them.  The array keeps whatever the last call left there; each
 * call writes every byte it reads before reading it, so nothing has to be
 * cleared between calls.
 *
 * Set-up: the first call on a device looks up that device's address of the
 * array (cudaGetSymbolAddress, with that device current), which may load the
 * library's module on that device; make that first call before any stream
 * capture.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 */
gdr_status gdr_chunk_fwd_segmented_noalloc(const void *q, const void *k, const void *v,
                                           gdr_dtype in_dtype, const float *g,
                                           gdr_gate_kind gate, const float *beta,
                                           const float *S0, void *o, float *S_T, int B, int T,
                                           int H, int dk, int dv, int C, int P,
                                           gdr_stream_t stream);

/*
 * The chunked forward over N packed sequences of different lengths (a
 * variable-length batch), one state per sequence and head.  Source as
 * gdr_chunk_fwd: each sequence runs the recurrence of "Decoding Hybrid
 * Linear Attention Architectures", sections 3 and 5, from its own S0.
 *
 *   q, k        [total_T, H, dk]  in_dtype the sequences back to back
 *   v, o        [total_T, H, dv]  in_dtype
 *   g           [total_T, H] fp32 (scalar gate) or [total_T, H, dk] (per
 *               channel); beta [total_T, H] fp32
 *   cu_seqlens  device int32 [N + 1]: sequence i is tokens
 *               [cu_seqlens[i], cu_seqlens[i + 1]); non-decreasing from 0 to
 *               total_T (values outside [0, total_T] are clamped into it)
 *   S0, S_T     [N, H, dv, dk] fp32 or NULL, as in gdr_chunk_fwd (S0 may
 *               alias S_T); an empty sequence gets S_T = S0 (or 0)
 *
 * S_T feeds gdr_step directly (same layout): prefill, then decode.  Any
 * shape gdr_chunk_fwd takes (bf16 with dk = dv = 128 on the
 * warp-specialised kernel, the rest on the split-operand kernel).  One
 * launch; no workspace.
 */
gdr_status gdr_chunk_fwd_varlen(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                                const float *g, gdr_gate_kind gate, const float *beta,
                                const int *cu_seqlens, const float *S0, void *o, float *S_T,
                                int N, int total_T, int H, int dk, int dv, int C,
                                gdr_stream_t stream);

/*
 * Chunked forward of gated linear attention, the delta rule's additive
 * sibling: "Decoding Hybrid Linear Attention Architectures", section 3 item
 * 4, and "Linear Attention Variants", gated linear attention:
 *
 *   S_t = S_{t-1} Diag(alpha_t) + v_t k_t^T,   o_t = S_t q_t,
 *
 * alpha_t = e^{g_t} (one value per head, or one per key channel), with no
 * erase term and no beta.  Computed chunkwise as gdr_chunk_fwd with the
 * correction W S dropped (T = I).
 *
 *   q, k   [B, T, H, dk] in_dtype;  v, o [B, T, H, dv] in_dtype
 *   g      [B, T, H] fp32 (scalar gate) or [B, T, H, dk] (per channel)
 *   S0     [B, H, dv, dk] fp32 or NULL (zero state); may alias S_T
 *   S_T    [B, H, dv, dk] fp32 or NULL (not written)
 *
 * Any shape gdr_chunk_fwd takes, C = 64 (GDR_ERR_UNSUPPORTED otherwise):
 * bf16 with dk = dv = 128 runs the warp-specialised kernel, the rest the
 * split-operand kernel.  T = 0 copies S0 (or zeros) to S_T.  One launch on
 * `stream`, no workspace; o must not alias an input.
 */
gdr_status gdr_chunk_fwd_gla(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                             const float *g, gdr_gate_kind gate, const float *S0, void *o,
                             float *S_T, int B, int T, int H, int dk, int dv, int C,
                             gdr_stream_t stream);

/* Bits of gdr_chunk_fwd_prologue's norm_qk. */
#define GDR_NORM_Q 1
#define GDR_NORM_K 2

/*
 * The chunked forward from raw projections: the prologue runs inside the
 * kernel, so the normalised q, k and the gates never go through HBM.
 * "Decoding Hybrid Linear Attention Architectures", section 3 item 2 (the
 * erase is a projector along a unit key), section 4 (beta in (0, 1), alpha
 * a forgetting rate in (0, 1]) and section 5 (gates in log space):
 *
 *   q <- q / sqrt(|q|^2 + 1e-6)   if norm_qk & GDR_NORM_Q   (per token, head)
 *   k <- k / sqrt(|k|^2 + 1e-6)   if norm_qk & GDR_NORM_K
 *   beta = 1 / (1 + e^{-b}),   g = log alpha = -gate_scale[h] * softplus(a)
 *
 * then the recurrence of gdr_chunk_fwd.
 *
 *   q, k        [B, T, H, dk] in_dtype  raw (not normalised) projections
 *   v, o        [B, T, H, dv] in_dtype
 *   a           [B, T, H] fp32 (scalar gate) or [B, T, H, dk] (per channel)
 *               gate logits;  b [B, T, H] fp32 write-strength logits
 *   gate_scale  [H] fp32, > 0        per-head decay scale
 *   S0, S_T     as gdr_chunk_fwd
 *
 * Any shape gdr_chunk_fwd takes, C = 64 (GDR_ERR_UNSUPPORTED otherwise):
 * bf16 with dk = dv = 128 and a scalar gate runs the warp-specialised
 * kernel; fp32 inputs, other head dims and per-channel gates (with the
 * range limit of gdr_chunk_fwd) run the split-operand kernel.  One launch,
 * no workspace (long sequences with few heads are not split into segments
 * on this entry).  The inputs are not modified.
 */
gdr_status gdr_chunk_fwd_prologue(const void *q, const void *k, const void *v,
                                  gdr_dtype in_dtype, const float *a, gdr_gate_kind gate,
                                  const float *gate_scale, const float *b, const float *S0,
                                  void *o, float *S_T, int B, int T, int H, int dk, int dv, int C,
                                  int norm_qk, gdr_stream_t stream);

/*
 * Diagonal-plus-low-rank (DPLR) transition, the generalised sibling of the
 * delta rule: "Decoding Hybrid Linear Attention Architectures", section 3
 * item 5:
 *
 *   S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,   o_t = S_t q_t
 *
 * (alpha_t = e^{g_t}, one per head or one per key channel; with
 * a = -beta (alpha . k), b = k and beta v it is the gated delta rule).
 *
 *   q, k, a, b  [B, T, H, dk] in_dtype;  v, o [B, T, H, dv] in_dtype
 *   g           [B, T, H] or [B, T, H, dk] fp32
 *   S0, S_T     [B, H, dv, dk] fp32 or NULL (zero state / not written)
 *
 * Chunked on the tensor cores (C = 64, one CTA per (b, h), one launch, no
 * workspace), the way section 5 of that page chunks the delta rule: per
 * chunk the low-rank reads x_r = S_{r-1} a_r solve a unit lower-triangular
 * system (the delta rule's WY form with the erase direction b and the write
 * key k kept apart), then o and the end state follow from three intra-chunk
 * products and two state products.  Operands are carried as two bf16 terms
 * and products as three MMAs (close to fp32 accuracy); the state is fp32.
 * dk, dv in {32, 64, 128} (GDR_ERR_UNSUPPORTED otherwise); pointers 16-byte
 * aligned; S0 may alias S_T.  A per-channel gate has the split-operand
 * range of gdr_chunk_fwd (decay over each half chunk above about -69 per
 * channel), beyond which the call records GDR_ERR_RANGE.
 */
gdr_status gdr_dplr_fwd(const void *q, const void *k, const void *v, const void *a,
                        const void *b, gdr_dtype in_dtype, const float *g, gdr_gate_kind gate,
                        const float *S0, void *o, float *S_T, int B, int T, int H, int dk,
                        int dv, gdr_stream_t stream);

/*
 * Backward of the chunked forward (training): the gradients of q, k, v,
 * g = log alpha, beta and S0 from dL/do and dL/dS_T.  "Decoding Hybrid
 * Linear Attention Architectures", section 5: backpropagation through the
 * same recurrence, with recomputation.  Per step (S' = S_{t-1} Diag(alpha),
 * p = S' k, u = beta (v - p), S_t = S' + u k^T, o = S_t q) and G = dL/dS_t:
 *
 *   G += do q^T;  dq = S_t^T do;  du = G k;  dbeta = du . (v - p);
 *   dv = beta du;  dk = G^T u - beta S'^T du;  dS' = G - beta du k^T;
 *   dg_j = sum_i S'[i][j] dS'[i][j] (summed over j for a scalar gate);
 *   G <- dS' Diag(alpha);  dS0 = G at the start.
 *
 *   q, k, v, g, beta, S0   as gdr_chunk_fwd (S0 NULL: zero)
 *   dout   [B, T, H, dv] fp32   dL/do
 *   dS_T   [B, H, dv, dk] fp32 or NULL (zero)
 *   dq, dk [B, T, H, dk] fp32;  dv [B, T, H, dv] fp32 (written)
 *   dg     [B, T, H] fp32 (scalar gate) or [B, T, H, dk] (per channel)
 *   dbeta  [B, T, H] fp32;  dS0 [B, H, dv, dk] fp32 or NULL (not written)
 *   workspace  device memory of gdr_chunk_bwd_workspace_bytes() bytes for
 *              the same shape, dtype and gate, 16-byte aligned, owned by the
 *              caller (overwritten)
 *
 * Two paths, chosen by shape:
 * - bf16 inputs, dk = dv = 128, scalar gate, T > 0: the chunked backward on
 *   the tensor cores (tcgen05), as section 5 has it (chunked and
 *   parallelised, with recomputation), in three launches: the forward again,
 *   stashing per chunk its start state, V'^T and T (bf16); a reverse pass
 *   over the chunks of each (b, h) carrying dL/dS in fp32 (stashing it and
 *   dV'^T per chunk, and writing dS0); a chunk-parallel pass forming dq,
 *   dk, dv, dg and dbeta.  Workspace: 104 KB per 64-token chunk and head.
 * - any other shape (dk = dv in {32, 64, 128}, fp32 or bf16 inputs, scalar
 *   or per-channel gate, T >= 0): the per-step reverse recurrence above in
 *   fp32 on CUDA cores, one CTA per (b, h), with the state checkpointed every
 *   8 tokens (workspace: those states and an 8-token stash per (b, h)); one
 *   launch.
 * GDR_ERR_UNSUPPORTED for dk != dv or a head size outside {32, 64, 128}.
 */
size_t gdr_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype in_dtype,
                                     gdr_gate_kind gate);
gdr_status gdr_chunk_bwd(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                         const float *g, gdr_gate_kind gate, const float *beta, const float *S0,
                         const float *dout, const float *dS_T, float *dq, float *dk, float *dv,
                         float *dg, float *dbeta, float *dS0, int B, int T, int H, int dk_,
                         int dv_, void *workspace, size_t ws_bytes, gdr_stream_t stream);

/*
 * One recurrent decode step for N independent states, S updated in place.
 * Source: "Decoding Hybrid Linear Attention Architectures", section 6
 * (constant-cost update of the fixed-size state per decoded token) with the
 * step order of section 3 item 6.
 *
 *   q, k  [N, H, dk]     in_dtype
 *   v     [N, H, dv]     in_dtype
 *   g     [N, H] or [N, H, dk]  fp32   log alpha (scalar / per-channel gate)
 *   beta  [N, H]         fp32
 *   S     [N, H, dv, dk] fp32          state, read and overwritten
 *   o     [N, H, dv]     in_dtype      output (written)
 *
 * o must not alias S or any input.
 */
gdr_status gdr_step(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                    const float *g, gdr_gate_kind gate, const float *beta, float *S, void *o,
                    int N, int H, int dk, int dv, gdr_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word.
 * Returns GDR_OK, GDR_ERR_TIMEOUT (a kernel gave up a bounded wait since the
 * last call), GDR_ERR_RANGE (a per-channel gate decayed beyond the
 * tensor-core path's range in some chunk since the last call; a time-out
 * takes precedence when both happened) or GDR_ERR_CUDA (the
 * synchronisation itself failed).
 */
gdr_status gdr_get_device_status(gdr_stream_t stream);

/* Static, human-readable name of a status code. */
const char *gdr_status_string(gdr_status s);

/* Detail of the last error returned on this host thread ("" if none). */
const char *gdr_last_error_message(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
