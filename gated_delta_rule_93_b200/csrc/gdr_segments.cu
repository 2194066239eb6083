// Long sequences with few (b, h): the sequence is cut into P equal segments
// that run as separate (b, h) units of the tensor-core chunked forward, so
// that B * H * P CTAs share the work of B * H.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5: the
// state after a stretch of tokens is linear in the state before it,
//   S_end = S_start M + E,
// M = the product of the per-token transitions (decay times I - beta k k^T)
// over the stretch, E = the state the stretch writes from a zero start.  The
// section applies this per chunk; here it is applied per segment:
//   pass 1a: every segment from zero (the first from S0): E_p, and for the
//            first segment its true end state;
//   pass 1b: every segment from the identity with v taken as zero: end state
//            M_p (d_v = d_k), the transition itself, with no difference of
//            two runs (which loses M_p's precision when it is not small);
//   combine: S_start(1) = end of segment 0, S_start(p + 1) = S_start(p) M_p +
//            E_p, in fp32; the last product is the final state S_T;
//   pass 2:  every segment from its true start state: the output o.
// The passes reuse the kernel on the same tensors, read as packed rows: segment
// p of sequence b is unit b * P + p, chunks [p nc / P, (p + 1) nc / P) of the
// sequence's nc chunks (so P need not divide them).
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kDim = 128;                   // d_k = d_v of the tensor-core kernel
constexpr int kRows = 16;                   // state rows per combine CTA
constexpr int kRowBlocks = kDim / kRows;
constexpr int kCombineThreads = 256;        // 4 row groups x 64 column pairs
// M, E_a of the current segment and the running rows
constexpr size_t kCombineSmem = (size_t)(2 * kDim * kDim + kRows * kDim) * sizeof(float);

// 16-byte global -> shared copy that bypasses the registers (many in flight
// per thread), and the wait for all of this thread's copies.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// One CTA per (b, h) and block of 16 state rows (rows of S are independent
// under S <- S M + E).  E_a: end states of pass 1a, E_b: of pass 1b (the
// transitions M_p), X: the
// start state of every segment (written), S_T: the final state (optional),
// all [B * P, H, 128, 128] except S0 / S_T [B, H, 128, 128] (S0 may alias
// S_T, so neither is declared __restrict__).  Each thread
// forms 4 rows x 2 columns of the product (a warp shares its rows), so every
// column pair of M read from shared memory serves four rows.
__global__ void __launch_bounds__(kCombineThreads)
    combine_segments(const float *S0, const float *__restrict__ Ea,
                     const float *__restrict__ Eb, float *__restrict__ X, float *S_T, int H,
                     int P) {
  extern __shared__ float smem[];
  float *M = smem;                    // [128][128] transition of the current segment
  float *MA = smem + kDim * kDim;     // [128][128] its E_a
  float *R = smem + 2 * kDim * kDim;  // [16][128] rows of the running start state
  const int bh = blockIdx.x, b = bh / H, h = bh % H, r0 = blockIdx.y * kRows;
  const int t = threadIdx.x;
  const size_t st = (size_t)kDim * kDim;
  auto seg = [&](int p) { return ((size_t)(b * P + p) * H + h) * st; };

  // segment 0 starts from S0 (or 0); segment 1 from segment 0's end state
#pragma unroll
  for (int j = 0; j < kRows * kDim / 4 / kCombineThreads; ++j) {
    const int i = t + j * kCombineThreads;  // float4 index in the row block
    const size_t off = (size_t)r0 * kDim + 4 * i;
    const float4 s0 = S0 ? *reinterpret_cast<const float4 *>(S0 + (size_t)bh * st + off)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 e0 = *reinterpret_cast<const float4 *>(Ea + seg(0) + off);
    *reinterpret_cast<float4 *>(X + seg(0) + off) = s0;
    *reinterpret_cast<float4 *>(X + seg(1) + off) = e0;
    reinterpret_cast<float4 *>(R)[i] = e0;
  }
  const int rg = t >> 6, c0 = (t & 63) * 2;  // rows 4 rg .. 4 rg + 3, columns c0, c0 + 1
  for (int p = 1; p < P; ++p) {
    __syncthreads();  // R written, M free
    const float4 *ea4 = reinterpret_cast<const float4 *>(Ea + seg(p));
    const float4 *eb4 = reinterpret_cast<const float4 *>(Eb + seg(p));
    float4 *m4 = reinterpret_cast<float4 *>(M), *a4 = reinterpret_cast<float4 *>(MA);
    // M = E_b and E_a of the segment into shared memory, every copy in
    // flight at once
#pragma unroll 8
    for (int j = 0; j < kDim * kDim / 4 / kCombineThreads; ++j) {
      const int i = t + j * kCombineThreads;
      cp_async16(m4 + i, eb4 + i);
      cp_async16(a4 + i, ea4 + i);
    }
    cp_async_wait_all();
    __syncthreads();
    float2 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      acc[i] = *reinterpret_cast<const float2 *>(MA + (size_t)(r0 + 4 * rg + i) * kDim + c0);
#pragma unroll 8
    for (int k = 0; k < kDim; ++k) {
      const float2 m = *reinterpret_cast<const float2 *>(M + k * kDim + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float s = R[(4 * rg + i) * kDim + k];
        acc[i].x = fmaf(s, m.x, acc[i].x);
        acc[i].y = fmaf(s, m.y, acc[i].y);
      }
    }
    __syncthreads();  // every thread has read R
    float *dst = nullptr;
    if (p + 1 < P)
      dst = X + seg(p + 1);
    else if (S_T)
      dst = S_T + (size_t)bh * st;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = 4 * rg + i;
      *reinterpret_cast<float2 *>(R + rr * kDim + c0) = acc[i];
      if (dst) *reinterpret_cast<float2 *>(dst + (size_t)(r0 + rr) * kDim + c0) = acc[i];
    }
  }
}

}  // namespace

int chunk_segments(const ChunkArgs &a, int num_sms) {
  if (!chunk_tc_supports(a) || a.dk != kDim || a.dv != kDim || a.skip_stage_chunk >= 0)
    return 1;
  const long long bh = (long long)a.B * a.H;
  if (bh <= 0 || num_sms <= 0 || (long long)a.B * a.T > 0x7fffffffLL) return 1;
  // Largest P with B * H * P CTAs in one wave and at least 16 chunks per
  // segment (segments of whole chunks, as even as that allows); three passes
  // pay off only from P = 4.
  const long long nc = ((long long)a.T + 63) / 64;
  int P = 1;
  while (P < 64 && bh * (P + 1) <= num_sms && nc / (P + 1) >= 16) ++P;
  return P >= 4 ? P : 1;
}

size_t chunk_segments_ws_bytes(const ChunkArgs &a, int P) {
  if (P <= 1) return 0;
  // X, E_a, E_b: one fp32 state per segment and head each
  return 3 * (size_t)a.B * P * a.H * a.dv * a.dk * sizeof(float);
}

cudaError_t launch_chunk_segments(const ChunkArgs &a, int P, void *ws, cudaStream_t stream) {
  static bool smem_set[64] = {};  // per device
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!smem_set[dev]) {
    e0 = cudaFuncSetAttribute(combine_segments, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kCombineSmem);
    if (e0 != cudaSuccess) return e0;
    smem_set[dev] = true;
  }
  const size_t n_state = (size_t)a.B * P * a.H * a.dv * a.dk;
  float *X = static_cast<float *>(ws), *Ea = X + n_state, *Eb = Ea + n_state;
  if ((long long)a.B * a.T > 0x7fffffffLL || P < 1) return cudaErrorInvalidValue;
  // the passes read the [B, T] tensors as packed rows, segment p of
  // sequence b being unit b * P + p (whole chunks, as even as they go)
  ChunkArgs s = a;
  s.B = a.B * P;
  s.T = a.B * a.T;
  s.seg_n = P;
  s.seg_T = a.T;
  // pass 1a: zero start (the first segment of a sequence from S0), end states
  s.S0 = a.S0;
  s.s0_seg = P;
  s.s0_identity = 0;
  s.S_T = Ea;
  s.o = nullptr;
  s.write_o = 0;
  cudaError_t e = launch_chunk_tc(s, stream);
  if (e != cudaSuccess) return e;
  // pass 1b: identity start with v taken as zero, end states = transitions
  s.S0 = nullptr;
  s.s0_seg = 0;
  s.s0_identity = 1;
  s.zero_v = 1;
  s.S_T = Eb;
  e = launch_chunk_tc(s, stream);
  if (e != cudaSuccess) return e;
  s.zero_v = 0;
  combine_segments<<<dim3(a.B * a.H, kRowBlocks), kCombineThreads, kCombineSmem, stream>>>(
      a.S0, Ea, Eb, X, a.S_T, a.H, P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // pass 2: every segment from its true start state; the output
  s.S0 = X;
  s.s0_identity = 0;
  s.S_T = nullptr;
  s.o = a.o;
  s.write_o = 1;
  return launch_chunk_tc(s, stream);
}

}  // namespace gdr
