// Diagonal-plus-low-rank (DPLR) transition, the generalised sibling of the
// delta rule, as a recurrent forward on CUDA cores (fp32 state):
//
//     S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,    o_t = S_t q_t
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 3 item 5.
// Per row i of S (value channel) the step is
//     x_i = S_i . a;   S_i <- S_i Diag(alpha) + x_i b^T + v_i k^T,
// and o_i = S_i . q after it, which expands to
//     o_i = S_{i,old} . (alpha q) + x_i (b . q) + v_i (k . q),
// so both dot products with the old row (and the two token scalars b.q,
// k.q) come out of one interleaved warp reduction per token.
//
// One CTA per (b, h), 16 warps: warp w owns rows w, w + 16, ..., lane l the
// key channels l, l + 32, ...; the state stays in registers.  The token
// vectors of 32 tokens are staged in shared memory (fp32, coalesced loads by
// the whole CTA) and the outputs of those tokens are collected there and
// stored coalesced.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 32;

struct DplrArgs {
  const void *q, *k, *v, *a, *b;
  const float *g, *S0;
  void *o;
  float *S_T;
  int B, T, H, d, bf16, per_channel;
};

__device__ __forceinline__ float ld_x(const void *p, size_t i, int bf16) {
  if (bf16) return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(p)[i] << 16);
  return reinterpret_cast<const float *>(p)[i];
}

template <int NC, int RW>
__global__ void __launch_bounds__(kThreads, 1) gdr_dplr_kernel(DplrArgs p) {
  constexpr int D = NC * 32;
  constexpr int NR = 2 * RW + 2;  // values reduced per token
  // staged chunk: q, k, a, b, v, o [kChunk][D], g [kChunk][D or 1]
  extern __shared__ float smem[];
  float *sq = smem, *sk = sq + kChunk * D, *sa = sk + kChunk * D, *sb = sa + kChunk * D;
  float *sv = sb + kChunk * D, *so = sv + kChunk * D, *sg = so + kChunk * D;
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int bh = blockIdx.x, bb = bh / p.H, h = bh % p.H;
  const int T = p.T, H = p.H;
  const size_t SS = (size_t)D * D;
  auto sidx = [&](int r, int c) { return (size_t)(w + 16 * r) * D + l + 32 * c; };

  float S[RW][NC];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int c = 0; c < NC; ++c) S[r][c] = p.S0 ? p.S0[(size_t)bh * SS + sidx(r, c)] : 0.f;

  for (int t0 = 0; t0 < T; t0 += kChunk) {
    const int n = min(kChunk, T - t0);
    __syncthreads();  // the previous chunk's outputs are stored
    for (int i = tid; i < n * D; i += kThreads) {
      const int t = i / D, j = i - t * D;
      const size_t x = (((size_t)bb * T + t0 + t) * H + h) * D + j;
      sq[i] = ld_x(p.q, x, p.bf16);
      sk[i] = ld_x(p.k, x, p.bf16);
      sa[i] = ld_x(p.a, x, p.bf16);
      sb[i] = ld_x(p.b, x, p.bf16);
      sv[i] = ld_x(p.v, x, p.bf16);
      if (p.per_channel) sg[i] = p.g[x];
    }
    if (!p.per_channel)
      for (int t = tid; t < n; t += kThreads) sg[t] = p.g[((size_t)bb * T + t0 + t) * H + h];
    __syncthreads();
    for (int t = 0; t < n; ++t) {
      float al[NC], kk[NC], bq[NC], aa[NC], vr[RW];
      float red[NR];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int j = t * D + l + 32 * c;
        al[c] = __expf(p.per_channel ? sg[j] : sg[t]);
        kk[c] = sk[j];
        aa[c] = sa[j];
        bq[c] = sb[j];
      }
#pragma unroll
      for (int r = 0; r < RW; ++r) vr[r] = sv[t * D + w + 16 * r];
      // partial sums: S_i . a, S_i . (alpha q) per row; b . q and k . q
      float pbq = 0.f, pkq = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float qc = sq[t * D + l + 32 * c];
        pbq = fmaf(bq[c], qc, pbq);
        pkq = fmaf(kk[c], qc, pkq);
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          if (c == 0) red[r] = red[RW + r] = 0.f;
          red[r] = fmaf(S[r][c], aa[c], red[r]);
          red[RW + r] = fmaf(S[r][c], al[c] * qc, red[RW + r]);
        }
      }
      red[2 * RW] = pbq;
      red[2 * RW + 1] = pkq;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int i = 0; i < NR; ++i) red[i] += __shfl_xor_sync(0xffffffffu, red[i], off);
      const float sbq = red[2 * RW], skq = red[2 * RW + 1];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const float x = red[r];
#pragma unroll
        for (int c = 0; c < NC; ++c)
          S[r][c] = fmaf(S[r][c], al[c], fmaf(x, bq[c], vr[r] * kk[c]));
        if (l == r) so[t * D + w + 16 * r] = red[RW + r] + x * sbq + vr[r] * skq;
      }
    }
    __syncthreads();
    for (int i = tid; i < n * D; i += kThreads) {
      const int t = i / D, j = i - t * D;
      const size_t x = (((size_t)bb * T + t0 + t) * H + h) * D + j;
      if (p.bf16)
        reinterpret_cast<__nv_bfloat16 *>(p.o)[x] = __float2bfloat16_rn(so[i]);
      else
        reinterpret_cast<float *>(p.o)[x] = so[i];
    }
  }
  if (p.S_T) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) p.S_T[(size_t)bh * SS + sidx(r, c)] = S[r][c];
  }
}

}  // namespace

cudaError_t launch_dplr(const void *q, const void *k, const void *v, const void *a,
                        const void *b, int bf16, const float *g, int per_channel,
                        const float *S0, void *o, float *S_T, int B, int T, int H, int d,
                        cudaStream_t stream) {
  DplrArgs p{q, k, v, a, b, g, S0, o, S_T, B, T, H, d, bf16, per_channel};
  const unsigned grid = (unsigned)((size_t)B * H);
  const size_t smem = ((size_t)6 * kChunk * d + (size_t)kChunk * (per_channel ? d : 1)) *
                      sizeof(float);
  auto go = [&](auto kern) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  };
  switch (d) {
    case 32: return go(gdr_dplr_kernel<1, 2>);
    case 64: return go(gdr_dplr_kernel<2, 4>);
    case 128: return go(gdr_dplr_kernel<4, 8>);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdr
