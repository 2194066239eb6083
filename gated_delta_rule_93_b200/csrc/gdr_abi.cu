// C ABI of the gated delta-rule library: argument validation, dispatch to
// the kernels, status reporting.  See include/gdr.h for the contract.
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "gdr_internal.cuh"
#include "gdr_testing.h"

namespace gdr {
__device__ unsigned int g_device_status = 0;
}

namespace {

thread_local char t_msg[512] = "";
thread_local int t_skip_stage_chunk = -1;  // testing hook, consumed by the next call

gdr_status fail(gdr_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof t_msg, fmt, ap);
  va_end(ap);
  return s;
}

gdr_status ok() {
  t_msg[0] = '\0';
  return GDR_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

gdr_status from_cuda(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return ok();
  return fail(GDR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Number of SMs of the current device (cached per device; 0 if unknown).
int device_sms() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

// The arguments as the kernels see them (no pointers).
gdr::ChunkArgs chunk_shape(int B, int T, int H, int dk, int dv, gdr_dtype in_dtype,
                           gdr_gate_kind gate) {
  gdr::ChunkArgs a{};
  a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv;
  a.bf16 = in_dtype == GDR_BF16;
  a.per_channel = gate == GDR_GATE_PER_CHANNEL;
  a.skip_stage_chunk = -1;
  a.s0_seg = 0;
  a.s0_identity = 0;
  a.write_o = 1;
  return a;
}

// Segments per sequence for this problem on the current device (1: none).
int segments_for(int B, int T, int H, int dk, int dv, int C, gdr_dtype in_dtype,
                 gdr_gate_kind gate) {
  if (B <= 0 || T <= 0 || H <= 0 || C != 64) return 1;
  if (in_dtype != GDR_F32 && in_dtype != GDR_BF16) return 1;
  if (gate != GDR_GATE_SCALAR && gate != GDR_GATE_PER_CHANNEL) return 1;
  return gdr::chunk_segments(chunk_shape(B, T, H, dk, dv, in_dtype, gate), device_sms());
}

// Device address of the status word on the current device (cached per device).
cudaError_t status_word(unsigned int **out) {
  static unsigned int *cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!cache[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, gdr::g_device_status);
    if (e != cudaSuccess) return e;
    cache[dev] = static_cast<unsigned int *>(p);
  }
  *out = cache[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

int gdr_version(void) { return 100; }

const char *gdr_status_string(gdr_status s) {
  switch (s) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
    case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
    case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT";
    case GDR_ERR_RANGE: return "GDR_ERR_RANGE";
  }
  return "GDR_ERR_UNKNOWN";
}

const char *gdr_last_error_message(void) { return t_msg; }

size_t gdr_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, int C,
                                     gdr_dtype in_dtype, gdr_gate_kind gate) {
  // Only the segment path of long sequences with few (b, h) needs scratch
  // (one fp32 state per segment and head, three sets); every kernel keeps its
  // intermediates on chip.
  const int P = segments_for(B, T, H, dk, dv, C, in_dtype, gate);
  return gdr::chunk_segments_ws_bytes(chunk_shape(B, T, H, dk, dv, in_dtype, gate), P);
}

int gdr_chunk_fwd_kernel_launches(int B, int T, int H, int dk, int dv, int C,
                                  gdr_dtype in_dtype, gdr_gate_kind gate) {
  if (B <= 0 || H <= 0 || T < 0) return 0;
  return segments_for(B, T, H, dk, dv, C, in_dtype, gate) > 1 ? 4 : 1;
}

}  // extern "C"

namespace {

// Checks shared by the chunked-forward entry points (everything but the
// workspace); fills the kernel arguments.  Returns GDR_OK or the error.
// (need_beta = false: beta is not read and may be null)
gdr_status check_chunk(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                       const float *g, gdr_gate_kind gate, const float *beta, const float *S0,
                       void *o, float *S_T, int B, int T, int H, int dk, int dv, int C,
                       gdr::ChunkArgs *out, bool need_beta = true) {
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "negative B/T/H");
  if (in_dtype != GDR_F32 && in_dtype != GDR_BF16)
    return fail(GDR_ERR_INVALID_ARG, "in_dtype must be GDR_F32 or GDR_BF16");
  if (gate != GDR_GATE_SCALAR && gate != GDR_GATE_PER_CHANNEL)
    return fail(GDR_ERR_INVALID_ARG, "unknown gate kind");
  if (C != 64) return fail(GDR_ERR_UNSUPPORTED, "chunk size C=%d (only 64 is built)", C);
  if (!head_dim_ok(dk) || !head_dim_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "head dims dk=%d dv=%d (need 32, 64 or 128)", dk, dv);
  if ((size_t)B * (size_t)H * (size_t)T > (size_t)1 << 40)
    return fail(GDR_ERR_INVALID_ARG, "problem too large");
  const bool empty_tokens = (size_t)B * H * T == 0;
  if (!empty_tokens) {
    if (!q || !k || !v || !g || (need_beta && !beta) || !o)
      return fail(GDR_ERR_INVALID_ARG, need_beta ? "null q/k/v/g/beta/o" : "null q/k/v/g/o");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) ||
        (need_beta && !aligned16(beta)) || !aligned16(o))
      return fail(GDR_ERR_INVALID_ARG, "q/k/v/g/beta/o must be 16-byte aligned");
  }
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
    return fail(GDR_ERR_INVALID_ARG, "S0/S_T must be 16-byte aligned");
  gdr::ChunkArgs a = chunk_shape(B, T, H, dk, dv, in_dtype, gate);
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S0 = S0; a.o = o; a.S_T = S_T;
  *out = a;
  return ok();
}

}  // namespace

extern "C" {

gdr_status gdr_chunk_fwd(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                         const float *g, gdr_gate_kind gate, const float *beta,
                         const float *S0, void *o, float *S_T, int B, int T, int H, int dk,
                         int dv, int C, void *workspace, size_t ws_bytes,
                         gdr_stream_t stream) {
  gdr::ChunkArgs a;
  gdr_status st = check_chunk(q, k, v, in_dtype, g, gate, beta, S0, o, S_T, B, T, H, dk, dv, C,
                              &a);
  if (st != GDR_OK) return st;
  const size_t need_ws = gdr_chunk_fwd_workspace_bytes(B, T, H, dk, dv, C, in_dtype, gate);
  if (ws_bytes < need_ws || (need_ws && !workspace))
    return fail(GDR_ERR_WORKSPACE, "workspace %zu B < required %zu B", ws_bytes, need_ws);
  if (need_ws && !aligned16(workspace))
    return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((size_t)B * H == 0) return ok();
  a.skip_stage_chunk = t_skip_stage_chunk;
  t_skip_stage_chunk = -1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd status word");
  // (an armed load-skip test hook keeps the single-pass kernel)
  const int P = a.skip_stage_chunk >= 0 ? 1 : segments_for(B, T, H, dk, dv, C, in_dtype, gate);
  if (P > 1)
    e = gdr::launch_chunk_segments(a, P, workspace, s);
  else if (gdr::chunk_tc_supports(a))
    e = gdr::launch_chunk_tc(a, s);
  else
    e = gdr::launch_chunk_split(a, s);
  return from_cuda(e, "gdr_chunk_fwd launch");
}

gdr_status gdr_chunk_fwd_segmented(const void *q, const void *k, const void *v,
                                   gdr_dtype in_dtype, const float *g, gdr_gate_kind gate,
                                   const float *beta, const float *S0, void *o, float *S_T,
                                   int B, int T, int H, int dk, int dv, int C, int P,
                                   void *workspace, size_t ws_bytes, gdr_stream_t stream) {
  gdr::ChunkArgs a;
  gdr_status st = check_chunk(q, k, v, in_dtype, g, gate, beta, S0, o, S_T, B, T, H, dk, dv, C,
                              &a);
  if (st != GDR_OK) return st;
  if (in_dtype != GDR_BF16 || dk != 128 || dv != 128)
    return fail(GDR_ERR_UNSUPPORTED, "segments need bf16 inputs and dk = dv = 128");
  if (P < 2 || T <= 0 || T % (64 * P) != 0)
    return fail(GDR_ERR_UNSUPPORTED, "P=%d segments of whole 64-token chunks (T=%d)", P, T);
  if ((size_t)B * P * H > (size_t)1 << 31) return fail(GDR_ERR_INVALID_ARG, "B*P*H too large");
  const size_t need_ws = gdr::chunk_segments_ws_bytes(a, P);
  if (ws_bytes < need_ws || !workspace)
    return fail(GDR_ERR_WORKSPACE, "workspace %zu B < required %zu B", ws_bytes, need_ws);
  if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((size_t)B * H == 0) return ok();
  a.skip_stage_chunk = -1;
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_segmented status word");
  return from_cuda(gdr::launch_chunk_segments(a, P, workspace,
                                              reinterpret_cast<cudaStream_t>(stream)),
                   "gdr_chunk_fwd_segmented launch");
}

// The segment path with its scratch in the library's fixed array instead of
// a caller's workspace, for callers that cannot allocate device memory when
// they run the mixer (see gdr.h).  Validation as gdr_chunk_fwd_segmented;
// sizes beyond the array are refused before anything touches the device.
gdr_status gdr_chunk_fwd_segmented_noalloc(const void *q, const void *k, const void *v,
                                           gdr_dtype in_dtype, const float *g,
                                           gdr_gate_kind gate, const float *beta,
                                           const float *S0, void *o, float *S_T, int B, int T,
                                           int H, int dk, int dv, int C, int P,
                                           gdr_stream_t stream) {
  gdr::ChunkArgs a;
  gdr_status st = check_chunk(q, k, v, in_dtype, g, gate, beta, S0, o, S_T, B, T, H, dk, dv, C,
                              &a);
  if (st != GDR_OK) return st;
  if (in_dtype != GDR_BF16 || dk != 128 || dv != 128)
    return fail(GDR_ERR_UNSUPPORTED, "segments need bf16 inputs and dk = dv = 128");
  if (P < 2 || T <= 0 || T % (64 * P) != 0)
    return fail(GDR_ERR_UNSUPPORTED, "P=%d segments of whole 64-token chunks (T=%d)", P, T);
  if ((size_t)B * P * H > (size_t)1 << 31) return fail(GDR_ERR_INVALID_ARG, "B*P*H too large");
  const size_t need = gdr::chunk_segments_ws_bytes(a, P);
  if (need > (size_t)GDR_NOALLOC_SCRATCH_BYTES)
    return fail(GDR_ERR_WORKSPACE,
                "needs %zu B of scratch (B*P*H = %zu segment-heads); the library's fixed array "
                "holds %zu B (B*P*H <= %zu)",
                need, (size_t)B * P * H, (size_t)GDR_NOALLOC_SCRATCH_BYTES,
                (size_t)GDR_NOALLOC_SCRATCH_BYTES / (3 * (size_t)dv * dk * sizeof(float)));
  if ((size_t)B * H == 0) return ok();
  a.skip_stage_chunk = -1;
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_segmented_noalloc status word");
  void *scratch = nullptr;
  e = gdr::noalloc_scratch(&scratch);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_segmented_noalloc scratch address");
  return from_cuda(gdr::launch_chunk_segments(a, P, scratch,
                                              reinterpret_cast<cudaStream_t>(stream)),
                   "gdr_chunk_fwd_segmented_noalloc launch");
}

gdr_status gdr_chunk_fwd_varlen(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                                const float *g, gdr_gate_kind gate, const float *beta,
                                const int *cu_seqlens, const float *S0, void *o, float *S_T,
                                int N, int total_T, int H, int dk, int dv, int C,
                                gdr_stream_t stream) {
  if (N < 0) return fail(GDR_ERR_INVALID_ARG, "negative N");
  gdr::ChunkArgs a;
  gdr_status st = check_chunk(q, k, v, in_dtype, g, gate, beta, S0, o, S_T, 1, total_T, H, dk,
                              dv, C, &a);
  if (st != GDR_OK) return st;
  if ((size_t)N * H == 0) return ok();
  if (!cu_seqlens) return fail(GDR_ERR_INVALID_ARG, "null cu_seqlens");
  if ((size_t)N * H > 0x7fffffffu) return fail(GDR_ERR_INVALID_ARG, "N*H too large");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_varlen status word");
  if (total_T == 0) {  // every sequence is empty: S_T = S0 (or 0)
    const size_t bytes = (size_t)N * H * dv * dk * sizeof(float);
    if (S_T && S0 && S_T != S0)
      e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s);
    else if (S_T && !S0)
      e = cudaMemsetAsync(S_T, 0, bytes, s);
    return from_cuda(e, "gdr_chunk_fwd_varlen copy");
  }
  a.B = N;
  a.cu_seqlens = cu_seqlens;
  return from_cuda(gdr::chunk_tc_supports(a) ? gdr::launch_chunk_tc(a, s)
                                             : gdr::launch_chunk_split(a, s),
                   "gdr_chunk_fwd_varlen launch");
}

gdr_status gdr_chunk_fwd_gla(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                             const float *g, gdr_gate_kind gate, const float *S0, void *o,
                             float *S_T, int B, int T, int H, int dk, int dv, int C,
                             gdr_stream_t stream) {
  gdr::ChunkArgs a;
  gdr_status st = check_chunk(q, k, v, in_dtype, g, gate, nullptr, S0, o, S_T, B, T, H, dk, dv,
                              C, &a, false);
  if (st != GDR_OK) return st;
  if ((size_t)B * H == 0) return ok();
  if ((size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_INVALID_ARG, "B*H too large");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_gla status word");
  if (T == 0) {  // no tokens: S_T = S0 (or 0)
    const size_t bytes = (size_t)B * H * dv * dk * sizeof(float);
    if (S_T && S0 && S_T != S0)
      e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s);
    else if (S_T && !S0)
      e = cudaMemsetAsync(S_T, 0, bytes, s);
    return from_cuda(e, "gdr_chunk_fwd_gla copy");
  }
  a.beta = nullptr;
  a.additive = 1;
  return from_cuda(gdr::chunk_tc_supports(a) ? gdr::launch_chunk_tc(a, s)
                                             : gdr::launch_chunk_split(a, s),
                   "gdr_chunk_fwd_gla launch");
}

gdr_status gdr_chunk_fwd_prologue(const void *q, const void *k, const void *v,
                                  gdr_dtype in_dtype, const float *a, gdr_gate_kind gate,
                                  const float *gate_scale, const float *b, const float *S0,
                                  void *o, float *S_T, int B, int T, int H, int dk, int dv, int C,
                                  int norm_qk, gdr_stream_t stream) {
  gdr::ChunkArgs ca;
  gdr_status st = check_chunk(q, k, v, in_dtype, a, gate, b, S0, o, S_T, B, T, H, dk, dv, C,
                              &ca);
  if (st != GDR_OK) return st;
  if (norm_qk < 0 || norm_qk > 3) return fail(GDR_ERR_INVALID_ARG, "norm_qk must be 0..3");
  if ((size_t)B * H == 0) return ok();
  if (!gate_scale) return fail(GDR_ERR_INVALID_ARG, "null gate_scale");
  if ((size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_INVALID_ARG, "B*H too large");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = status_word(&ca.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_fwd_prologue status word");
  if (T == 0) {  // no tokens: S_T = S0 (or 0)
    const size_t bytes = (size_t)B * H * dv * dk * sizeof(float);
    if (S_T && S0 && S_T != S0)
      e = cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s);
    else if (S_T && !S0)
      e = cudaMemsetAsync(S_T, 0, bytes, s);
    return from_cuda(e, "gdr_chunk_fwd_prologue copy");
  }
  ca.prologue = 1;
  ca.norm_qk = norm_qk;
  ca.gate_scale = gate_scale;
  // the warp-specialised kernel takes bf16, d = 128 with a scalar gate; every
  // other shape and per-channel gates run the split-operand kernel
  const bool tc = gdr::chunk_tc_supports(ca) && gate == GDR_GATE_SCALAR;
  ca.skip_stage_chunk = tc ? t_skip_stage_chunk : -1;
  t_skip_stage_chunk = -1;
  return from_cuda(tc ? gdr::launch_chunk_tc(ca, s) : gdr::launch_chunk_split(ca, s),
                   "gdr_chunk_fwd_prologue launch");
}

gdr_status gdr_dplr_fwd(const void *q, const void *k, const void *v, const void *a,
                        const void *b, gdr_dtype in_dtype, const float *g, gdr_gate_kind gate,
                        const float *S0, void *o, float *S_T, int B, int T, int H, int dk,
                        int dv, gdr_stream_t stream) {
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "negative B/T/H");
  if (in_dtype != GDR_F32 && in_dtype != GDR_BF16)
    return fail(GDR_ERR_INVALID_ARG, "in_dtype must be GDR_F32 or GDR_BF16");
  if (gate != GDR_GATE_SCALAR && gate != GDR_GATE_PER_CHANNEL)
    return fail(GDR_ERR_INVALID_ARG, "unknown gate kind");
  if (!head_dim_ok(dk) || !head_dim_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "DPLR head dims dk=%d dv=%d (need 32, 64 or 128)", dk, dv);
  if ((size_t)B * (size_t)H * (size_t)T > (size_t)1 << 40)
    return fail(GDR_ERR_INVALID_ARG, "problem too large");
  if ((size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_INVALID_ARG, "B*H too large");
  if ((size_t)B * H * T != 0) {
    if (!q || !k || !v || !a || !b || !g || !o)
      return fail(GDR_ERR_INVALID_ARG, "null q/k/v/a/b/g/o");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(b) ||
        !aligned16(g) || !aligned16(o))
      return fail(GDR_ERR_INVALID_ARG, "q/k/v/a/b/g/o must be 16-byte aligned");
  }
  if ((S0 && !aligned16(S0)) || (S_T && !aligned16(S_T)))
    return fail(GDR_ERR_INVALID_ARG, "S0/S_T must be 16-byte aligned");
  if ((size_t)B * H == 0) return ok();
  gdr::DplrChunkArgs p;
  p.q = q; p.k = k; p.v = v; p.a = a; p.b = b; p.g = g; p.S0 = S0; p.o = o; p.S_T = S_T;
  p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv;
  p.bf16 = in_dtype == GDR_BF16;
  p.per_channel = gate == GDR_GATE_PER_CHANNEL;
  cudaError_t e = status_word(&p.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_dplr_fwd status word");
  return from_cuda(gdr::launch_dplr_chunk(p, reinterpret_cast<cudaStream_t>(stream)),
                   "gdr_dplr_fwd launch");
}

namespace {
// The backward's path for a shape: the tensor-core chunked backward, or the
// per-step recurrence on CUDA cores.
bool bwd_on_tensor_cores(int T, int d, gdr_dtype in_dtype, gdr_gate_kind gate) {
  return T > 0 && gdr::bwd_tc_supports(in_dtype == GDR_BF16, gate == GDR_GATE_PER_CHANNEL, d);
}
}  // namespace

size_t gdr_chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype in_dtype,
                                     gdr_gate_kind gate) {
  if (dk != dv || (dk != 32 && dk != 64 && dk != 128)) return 0;
  if (bwd_on_tensor_cores(T, dk, in_dtype, gate)) return gdr::bwd_tc_ws_bytes(B, T, H);
  return gdr::bwd_ws_bytes(B, T, H, dk);
}

gdr_status gdr_chunk_bwd(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                         const float *g, gdr_gate_kind gate, const float *beta, const float *S0,
                         const float *dout, const float *dS_T, float *dq, float *dk, float *dv,
                         float *dg, float *dbeta, float *dS0, int B, int T, int H, int dk_,
                         int dv_, void *workspace, size_t ws_bytes, gdr_stream_t stream) {
  if (B < 0 || T < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "negative B/T/H");
  if (in_dtype != GDR_F32 && in_dtype != GDR_BF16)
    return fail(GDR_ERR_INVALID_ARG, "in_dtype must be GDR_F32 or GDR_BF16");
  if (gate != GDR_GATE_SCALAR && gate != GDR_GATE_PER_CHANNEL)
    return fail(GDR_ERR_INVALID_ARG, "unknown gate kind");
  if (dk_ != dv_ || (dk_ != 32 && dk_ != 64 && dk_ != 128))
    return fail(GDR_ERR_UNSUPPORTED, "backward needs dk = dv in {32, 64, 128} (got %d, %d)", dk_,
                dv_);
  if ((size_t)B * (size_t)H * (size_t)T > (size_t)1 << 40)
    return fail(GDR_ERR_INVALID_ARG, "problem too large");
  if ((size_t)B * H > 0x7fffffffu) return fail(GDR_ERR_INVALID_ARG, "B*H too large");
  if ((size_t)B * H * T != 0) {
    if (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta)
      return fail(GDR_ERR_INVALID_ARG, "null input or gradient pointer");
  }
  const size_t need = gdr_chunk_bwd_workspace_bytes(B, T, H, dk_, dv_, in_dtype, gate);
  if ((size_t)B * H != 0 && (ws_bytes < need || !workspace))
    return fail(GDR_ERR_WORKSPACE, "workspace %zu B < required %zu B", ws_bytes, need);
  if (workspace && !aligned16(workspace))
    return fail(GDR_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((size_t)B * H == 0) return ok();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bwd_on_tensor_cores(T, dk_, in_dtype, gate)) {
    if ((size_t)B * H * ((T + 63) / 64) > 0x7fffffffu)
      return fail(GDR_ERR_INVALID_ARG, "B*H*chunks too large");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout))
      return fail(GDR_ERR_INVALID_ARG, "q/k/v/dout must be 16-byte aligned");
    unsigned int *status = nullptr;
    cudaError_t e = status_word(&status);
    if (e != cudaSuccess) return from_cuda(e, "gdr_chunk_bwd status word");
    return from_cuda(gdr::launch_bwd_tc(q, k, v, g, beta, S0, dout, dS_T, dq, dk, dv, dg, dbeta,
                                        dS0, B, T, H, workspace, status, s),
                     "gdr_chunk_bwd launch (tensor cores)");
  }
  return from_cuda(gdr::launch_bwd(q, k, v, in_dtype == GDR_BF16, g, gate == GDR_GATE_PER_CHANNEL,
                                   beta, S0, dout, dS_T, dq, dk, dv, dg, dbeta, dS0, B, T, H,
                                   dk_, workspace, s),
                   "gdr_chunk_bwd launch");
}

gdr_status gdr_step(const void *q, const void *k, const void *v, gdr_dtype in_dtype,
                    const float *g, gdr_gate_kind gate, const float *beta, float *S, void *o,
                    int N, int H, int dk, int dv, gdr_stream_t stream) {
  if (N < 0 || H < 0) return fail(GDR_ERR_INVALID_ARG, "negative N/H");
  if (in_dtype != GDR_F32 && in_dtype != GDR_BF16)
    return fail(GDR_ERR_INVALID_ARG, "in_dtype must be GDR_F32 or GDR_BF16");
  if (gate != GDR_GATE_SCALAR && gate != GDR_GATE_PER_CHANNEL)
    return fail(GDR_ERR_INVALID_ARG, "unknown gate kind");
  if (!head_dim_ok(dk) || !head_dim_ok(dv))
    return fail(GDR_ERR_UNSUPPORTED, "head dims dk=%d dv=%d (need 32, 64 or 128)", dk, dv);
  if ((size_t)N * H == 0) return ok();
  if (!q || !k || !v || !g || !beta || !S || !o)
    return fail(GDR_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(beta) ||
      !aligned16(S) || !aligned16(o))
    return fail(GDR_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((size_t)N * H > (size_t)1 << 31) return fail(GDR_ERR_INVALID_ARG, "N*H too large");
  gdr::StepArgs a;
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.S = S; a.o = o;
  a.N = N; a.H = H; a.dk = dk; a.dv = dv;
  a.bf16 = in_dtype == GDR_BF16;
  a.per_channel = gate == GDR_GATE_PER_CHANNEL;
  cudaError_t e = status_word(&a.status);
  if (e != cudaSuccess) return from_cuda(e, "gdr_step status word");
  return from_cuda(gdr::launch_step(a, reinterpret_cast<cudaStream_t>(stream)),
                   "gdr_step launch");
}

gdr_status gdr_testing_skip_stage_load(int chunk) {
  if (chunk < 0) return fail(GDR_ERR_INVALID_ARG, "chunk must be >= 0");
  t_skip_stage_chunk = chunk;
  return ok();
}

gdr_status gdr_get_device_status(gdr_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int word = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&word, gdr::g_device_status, sizeof word, 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(gdr::g_device_status, &zero, sizeof zero, 0,
                                cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e, "gdr_get_device_status");
  if (word & gdr::kStatusTimeout)
    return fail(GDR_ERR_TIMEOUT, "a kernel gave up a bounded wait (status word 0x%x)", word);
  if (word & gdr::kStatusRange)
    return fail(GDR_ERR_RANGE,
                "a per-channel gate decayed beyond the tensor-core path's range (more than "
                "about 83 in log decay over half a chunk); those results are not valid "
                "(status word 0x%x)",
                word);
  return ok();
}

}  // extern "C"
