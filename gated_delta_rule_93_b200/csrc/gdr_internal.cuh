// Internal declarations shared by the gated delta-rule CUDA sources.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

// Kernels OR error bits into a device status word (they never trap).  The
// word lives in gdr_abi.cu; launchers receive its device address.
constexpr unsigned int kStatusTimeout = 1u;
// A per-channel gate decayed faster than the tensor-core path's tile scaling
// can represent in some chunk (that call's results are not the recurrence's).
constexpr unsigned int kStatusRange = 2u;

struct ChunkArgs {
  const void *q, *k, *v;
  const float *g;
  const float *beta;
  const float *S0;
  void *o;
  float *S_T;
  int B, T, H, dk, dv;
  int bf16;          // 1: q, k, v, o are bf16; 0: fp32
  int per_channel;   // 1: g is [B,T,H,dk]
  unsigned int *status;  // device status word
  int skip_stage_chunk;  // testing: chunk whose input load is never issued (-1: none)
  // Segment passes of a long sequence (tensor-core kernel only; 0 / 0 / 1
  // for an ordinary call):
  int s0_seg;       // > 0: sequence b reads S0[b / s0_seg] if b % s0_seg == 0, else starts at 0
  int s0_identity;  // 1: sequences without an S0 start from the identity (d_v == d_k)
  int zero_v;       // 1: v is taken as zero (not read): the end state is the transition
  int write_o;      // 0: o is not written (may be null)
  // Segment passes with uneven segments (tensor-core kernel only; 0: off):
  // the tensors are read as packed rows [1, total, H, d], and sequence
  // b is segment b % seg_n of original sequence b / seg_n (seg_T tokens),
  // chunks split as evenly as whole chunks allow; a.T is then the packed
  // total and a.B the number of segments.
  int seg_n, seg_T;
  // Packed sequences (tensor-core kernel only): B sequences, sequence b is
  // tokens [cu_seqlens[b], cu_seqlens[b + 1]) of the [1, T, H, d] tensors
  // (device int32 [B + 1]); null: dense [B, T, H, d].
  const int *cu_seqlens;
  // Additive writes (tensor-core kernel only): 1 runs gated linear attention,
  // S_t = S_{t-1} Diag(alpha_t) + v_t k_t^T, with beta unused (may be null).
  int additive;
  // Prologue (tensor-core kernel, scalar gates): 1 reads g as gate logits a
  // (g = -gate_scale[h] softplus(a)) and beta as logits b (beta = sigmoid(b))
  // and L2-normalises q (norm_qk & 1) and k (norm_qk & 2) in the kernel.
  int prologue;
  int norm_qk;
  const float *gate_scale;  // [H]
  // Stash for the backward (tensor-core kernel, scalar gates, write_o = 0):
  // per (b, h) and chunk c, in bf16, row-major: the state at the chunk's
  // start X0 = S_c [128][128] (value channel, key channel), V'^T [128][64]
  // (value channel, token) and T = (I + A)^{-1} Diag(beta) [64][64].
  // Null: nothing is stashed.
  __nv_bfloat16 *stash_x, *stash_v, *stash_t;
};

struct StepArgs {
  const void *q, *k, *v;
  const float *g;
  const float *beta;
  float *S;
  void *o;
  int N, H, dk, dv;
  int bf16;
  int per_channel;
  unsigned int *status;
};

// Launchers return cudaSuccess or the launch error.
cudaError_t launch_step(const StepArgs &a, cudaStream_t stream);
// Split-operand tensor-core forward (fp32 inputs, and head dims the
// warp-specialised kernel does not take): every operand as two bf16 terms,
// every product as three MMAs; returns cudaErrorNotSupported outside its
// shapes.
cudaError_t launch_chunk_split(const ChunkArgs &a, cudaStream_t stream);
bool chunk_split_supports(const ChunkArgs &a);
// Tensor-core (tcgen05) chunked forward; returns cudaErrorNotSupported when
// the shape is outside what it handles, so the caller can pick another path.
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream);
bool chunk_tc_supports(const ChunkArgs &a);
// Tensor maps of the tensor-core kernels (host): a [B, T, H, d] bf16 tensor
// in 64 x 64 boxes, and a per-chunk array [nchunks][rows][cols] bf16 in
// 64 x 64 boxes, both with the 128-byte swizzle.
bool tc_map_bf16(CUtensorMap *m, const void *base, int B, int T, int H, int d);
bool tc_map_stash(CUtensorMap *m, const void *base, long long nchunks, int rows, int cols);

// Long sequences with few (b, h): each sequence is cut into P segments that
// run as separate (b, h) units (two passes of the tensor-core kernel, a
// combine of the segments' states, a final pass).  P = 1: not used.
int chunk_segments(const ChunkArgs &a, int num_sms);
size_t chunk_segments_ws_bytes(const ChunkArgs &a, int P);
cudaError_t launch_chunk_segments(const ChunkArgs &a, int P, void *ws, cudaStream_t stream);
// Device address, on the current device, of the library's fixed scratch
// array (GDR_NOALLOC_SCRATCH_BYTES), looked up once per device.
cudaError_t noalloc_scratch(void **out);
// DPLR transition, chunked forward on the tensor cores (split operands):
// S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T, o_t = S_t q_t.
struct DplrChunkArgs {
  const void *q, *k, *v, *a, *b;  // [B, T, H, dk] (v: dv), bf16 or fp32
  const float *g;                 // [B, T, H] or [B, T, H, dk]
  const float *S0;                // [B, H, dv, dk] or null
  void *o;                        // [B, T, H, dv]
  float *S_T;                     // [B, H, dv, dk] or null
  int B, T, H, dk, dv;
  int bf16, per_channel;
  unsigned int *status;
};
cudaError_t launch_dplr_chunk(const DplrChunkArgs &a, cudaStream_t stream);
// Backward of the recurrence (CUDA cores, d_k = d_v = d in {32, 64, 128}).
size_t bwd_ws_bytes(int B, int T, int H, int d);
cudaError_t launch_bwd(const void *q, const void *k, const void *v, int bf16, const float *g,
                       int per_channel, const float *beta, const float *S0, const float *dout,
                       const float *dST, float *dq, float *dk, float *dv, float *dg,
                       float *dbeta, float *dS0, int B, int T, int H, int d, void *ws,
                       cudaStream_t stream);

// Backward on the tensor cores (bf16, d_k = d_v = 128, scalar gate): the
// forward rerun with a per-chunk stash, a reverse pass for the state
// gradient and a chunk-parallel pass for the token gradients (3 launches).
bool bwd_tc_supports(int bf16, int per_channel, int d);
size_t bwd_tc_ws_bytes(int B, int T, int H);
cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *S0, const float *dout,
                          const float *dST, float *dq, float *dk, float *dv, float *dg,
                          float *dbeta, float *dS0, int B, int T, int H, void *ws,
                          unsigned int *status, cudaStream_t stream);

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float load_in(const void *p, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ void store_out(void *p, size_t i, float x, int bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[i] = x;
}

}  // namespace gdr
