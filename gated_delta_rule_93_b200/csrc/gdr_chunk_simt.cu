// Chunkwise gated delta-rule forward on CUDA cores, all in fp32.
//
// This is the fp32-input path (fp32 inputs ask for 1e-4 agreement, which a
// bf16 tensor-core operand cannot give) and the fallback for shapes the
// tensor-core kernel does not take.  It follows the same chunk algorithm:
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5
// (inter-chunk state recursion, intra-chunk output, log-space gates) and the
// WY/UT form of the delta rule from "Linear Attention Variants (RetNet, GLA,
// DeltaNet, Based)", DeltaNet section.  In the kernel's orientation the
// state is X = S^T (d_k x d_v) and, for one chunk of C = 64 rows,
//   gc_r = sum_{s<=r} g_s           (cumulative log decay from chunk start)
//   A[r][s] = beta_r sum_j K[r][j] K[s][j] exp(gc_r[j] - gc_s[j])   (s < r)
//   P[r][s] =        sum_j Q[r][j] K[s][j] exp(gc_r[j] - gc_s[j])   (s <= r)
//   T = (I + A)^{-1} Diag(beta)                      (forward substitution)
//   W = T (K * e^{gc}),  U = T V
//   V' = U - W X
//   O  = (Q * e^{gc}) X + P V'
//   X <- Diag(e^{gc_last}) X + (K * e^{gc_last - gc})^T V'
// Every exponent is <= 0, so no intermediate can overflow for any gate.
//
// Grid: one CTA per (b, h, 32-column slice of d_v); the slice's columns of
// X are independent, the A/T/W work is repeated per slice.  256 threads.
// A ragged last chunk is zero-padded (k = q = v = 0, beta = 0, g = 0), which
// leaves the state untouched; its padded output rows are not stored.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int DK, int DVS, bool PERCH>
struct Smem {
  static constexpr int DKP = DK + 1;  // odd row stride: conflict-free columns
  static constexpr int CP = C + 1;
  // offsets in floats
  static constexpr int oX = 0;                   // X slice [DK][DVS]
  static constexpr int oK = oX + DK * DVS;       // K raw -> K_bar  [C][DKP]
  static constexpr int oQ = oK + C * DKP;        // Q raw -> Q~     [C][DKP]
  static constexpr int oKt = oQ + C * DKP;       // K~              [C][DKP]
  static constexpr int oG = oKt + C * DKP;       // gc [C][DKP] or [C], later W
  static constexpr int oT = oG + C * DKP;        // A -> T          [C][CP]
  static constexpr int oP = oT + C * CP;         // P               [C][CP]
  static constexpr int oV = oP + C * CP;         // V -> U -> V'    [C][DVS]
  static constexpr int oB = oV + C * DVS;        // beta [C]
  static constexpr int total = oB + C;
  static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <int DK, int DVS, bool BF16, bool PERCH>
__global__ void __launch_bounds__(kThreads, 1) gdr_chunk_simt_kernel(ChunkArgs a) {
  using L = Smem<DK, DVS, PERCH>;
  constexpr int DKP = L::DKP, CP = L::CP;
  extern __shared__ float sm[];
  float *X = sm + L::oX;
  float *Ks = sm + L::oK;
  float *Qs = sm + L::oQ;
  float *Kt = sm + L::oKt;
  float *G = sm + L::oG;
  float *Wm = sm + L::oG;  // reuses G once the scaled copies exist
  float *Tm = sm + L::oT;
  float *Pm = sm + L::oP;
  float *Vb = sm + L::oV;
  float *Bt = sm + L::oB;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nslices = a.dv / DVS;
  const int slice = blockIdx.x % nslices;
  const int bh = blockIdx.x / nslices;
  const int b = bh / a.H, h = bh % a.H;
  const int c0 = slice * DVS;
  const int T = a.T, H = a.H, dv = a.dv;

  // X = S0^T restricted to this slice (S0 is [dv][dk] per head).
  for (int idx = tid; idx < DK * DVS; idx += kThreads) {
    const int j = idx / DVS, i = idx % DVS;
    X[idx] = a.S0 ? a.S0[((size_t)bh * dv + c0 + i) * DK + j] : 0.f;
  }

  for (int t0 = 0; t0 < T; t0 += C) {
    const int Lr = min(C, T - t0);
    __syncthreads();  // previous chunk fully consumed
    // ---- load the chunk (zero-padded tail)
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int r = idx / DK, j = idx % DK;
      float kv = 0.f, qv = 0.f;
      if (r < Lr) {
        const size_t tok = ((size_t)b * T + t0 + r) * H + h;
        kv = load_in(a.k, tok * DK + j, BF16);
        qv = load_in(a.q, tok * DK + j, BF16);
      }
      Ks[r * DKP + j] = kv;
      Qs[r * DKP + j] = qv;
      if constexpr (PERCH) {
        G[r * DKP + j] = r < Lr ? a.g[(((size_t)b * T + t0 + r) * H + h) * DK + j] : 0.f;
      }
    }
    for (int idx = tid; idx < C * DVS; idx += kThreads) {
      const int r = idx / DVS, i = idx % DVS;
      float vv = 0.f;
      if (r < Lr) vv = load_in(a.v, (((size_t)b * T + t0 + r) * H + h) * dv + c0 + i, BF16);
      Vb[idx] = vv;
    }
    if (tid < C) {
      const int r = tid;
      const size_t tok = ((size_t)b * T + t0 + r) * H + h;
      Bt[r] = r < Lr ? a.beta[tok] : 0.f;
      if constexpr (!PERCH) G[r] = r < Lr ? a.g[tok] : 0.f;
    }
    __syncthreads();
    // ---- cumulative log decay within the chunk (log-space, fp32)
    if constexpr (PERCH) {
      for (int j = tid; j < DK; j += kThreads) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
          acc += G[r * DKP + j];
          G[r * DKP + j] = acc;
        }
      }
    } else {
      if (warp == 0) {
        float x0 = G[lane], x1 = G[lane + 32];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
          if (lane >= off) { x0 += y0; x1 += y1; }
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        G[lane] = x0;
        G[lane + 32] = x1;
      }
    }
    __syncthreads();
    // ---- A (strict) and P (inclusive) with exact pairwise decays
    for (int idx = tid; idx < C * C; idx += kThreads) {
      const int r = idx / C, s = idx % C;
      float accA = 0.f, accP = 0.f;
      if (s <= r) {
        if constexpr (PERCH) {
          for (int j = 0; j < DK; ++j) {
            const float d = __expf(G[r * DKP + j] - G[s * DKP + j]);
            const float ks = Ks[s * DKP + j] * d;
            accA += Ks[r * DKP + j] * ks;
            accP += Qs[r * DKP + j] * ks;
          }
        } else {
          for (int j = 0; j < DK; ++j) {
            accA += Ks[r * DKP + j] * Ks[s * DKP + j];
            accP += Qs[r * DKP + j] * Ks[s * DKP + j];
          }
          const float d = __expf(G[r] - G[s]);
          accA *= d;
          accP *= d;
        }
      }
      Tm[r * CP + s] = (s < r) ? Bt[r] * accA : 0.f;
      Pm[r * CP + s] = accP;  // zero above the diagonal
    }
    __syncthreads();
    // ---- scaled copies: K~ = K e^{gc}, Q~ = Q e^{gc}, K_bar = K e^{gc_last - gc}
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int r = idx / DK, j = idx % DK;
      const float gr = PERCH ? G[r * DKP + j] : G[r];
      const float gl = PERCH ? G[(C - 1) * DKP + j] : G[C - 1];
      const float kv = Ks[r * DKP + j];
      Kt[r * DKP + j] = kv * __expf(gr);
      Qs[r * DKP + j] *= __expf(gr);
      Ks[r * DKP + j] = kv * __expf(gl - gr);
    }
    // chunk-end decay per key channel, kept in registers of the X-update owner
    // (thread mapping of the X update below: j = warp + 8 m, i = lane)
    float dec_last[DK / kWarps];
#pragma unroll
    for (int m = 0; m < DK / kWarps; ++m) {
      const int j = warp + kWarps * m;
      dec_last[m] = __expf(PERCH ? G[(C - 1) * DKP + j] : G[C - 1]);
    }
    __syncthreads();
    // ---- T = (I + A)^{-1} Diag(beta), forward substitution in place, one row
    // at a time: Y_i = e_i - sum_{k<i} A[i][k] Y_k.  Four threads per column c
    // split the k-sum.  Row i still holds A while it is read; it is
    // overwritten with Y_i only after every thread has read it.
    {
      const int c = tid >> 2, part = tid & 3;
      for (int i = 1; i < C; ++i) {
        float acc = 0.f;
        if (c < i)
          for (int kk = c + part; kk < i; kk += 4) {
            const float y = (kk == c) ? 1.f : Tm[kk * CP + c];  // Y has a unit diagonal
            acc += Tm[i * CP + kk] * y;
          }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        __syncthreads();
        if (part == 0 && c < i) Tm[i * CP + c] = -acc;
        __syncthreads();
      }
      // unit diagonal, zero above; then scale column s by beta_s
      for (int idx = tid; idx < C * C; idx += kThreads) {
        const int r = idx / C, s2 = idx % C;
        const float y = (s2 < r) ? Tm[r * CP + s2] : (s2 == r ? 1.f : 0.f);
        Tm[r * CP + s2] = y * Bt[s2];
      }
    }
    __syncthreads();
    // ---- W = T K~   [C][DK]   (thread: j = lane + 32 jj, r = warp + 8 m)
    for (int m = 0; m < C / kWarps; ++m) {
      const int r = warp + kWarps * m;
#pragma unroll
      for (int jj = 0; jj < DK / 32; ++jj) {
        const int j = lane + 32 * jj;
        float acc = 0.f;
        for (int s2 = 0; s2 <= r; ++s2) acc += Tm[r * CP + s2] * Kt[s2 * DKP + j];
        Wm[r * DKP + j] = acc;
      }
    }
    __syncthreads();
    // ---- U = T V, then V' = U - W X   (thread: i = lane, r = warp + 8 m)
    float vp[C / kWarps];
#pragma unroll
    for (int m = 0; m < C / kWarps; ++m) {
      const int r = warp + kWarps * m, i = lane;
      float u = 0.f;
      for (int s2 = 0; s2 <= r; ++s2) u += Tm[r * CP + s2] * Vb[s2 * DVS + i];
      float wx = 0.f;
      for (int j = 0; j < DK; ++j) wx += Wm[r * DKP + j] * X[j * DVS + i];
      vp[m] = u - wx;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < C / kWarps; ++m) Vb[(warp + kWarps * m) * DVS + lane] = vp[m];
    __syncthreads();
    // ---- O = Q~ X + P V'   (rows < Lr are stored)
#pragma unroll
    for (int m = 0; m < C / kWarps; ++m) {
      const int r = warp + kWarps * m, i = lane;
      if (r < Lr) {
        float acc = 0.f;
        for (int j = 0; j < DK; ++j) acc += Qs[r * DKP + j] * X[j * DVS + i];
        for (int s2 = 0; s2 <= r; ++s2) acc += Pm[r * CP + s2] * Vb[s2 * DVS + i];
        const size_t tok = ((size_t)b * T + t0 + r) * H + h;
        store_out(a.o, tok * dv + c0 + i, acc, BF16);
      }
    }
    __syncthreads();
    // ---- X <- Diag(e^{gc_last}) X + K_bar^T V'   (thread: i = lane, j = warp + 8 m)
#pragma unroll
    for (int m = 0; m < DK / kWarps; ++m) {
      const int j = warp + kWarps * m, i = lane;
      float acc = dec_last[m] * X[j * DVS + i];
      for (int r = 0; r < C; ++r) acc += Ks[r * DKP + j] * Vb[r * DVS + i];
      X[j * DVS + i] = acc;
    }
  }
  __syncthreads();
  if (a.S_T) {
    for (int idx = tid; idx < DK * DVS; idx += kThreads) {
      const int j = idx / DVS, i = idx % DVS;
      a.S_T[((size_t)bh * dv + c0 + i) * DK + j] = X[idx];
    }
  }
}

template <int DK, bool BF16, bool PERCH>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t stream) {
  constexpr int DVS = 32;
  using L = Smem<DK, DVS, PERCH>;
  auto kern = gdr_chunk_simt_kernel<DK, DVS, BF16, PERCH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::bytes);
  if (e != cudaSuccess) return e;
  const size_t blocks = (size_t)a.B * a.H * (a.dv / DVS);
  if (blocks > 0x7fffffffu) return cudaErrorInvalidValue;
  kern<<<(unsigned)blocks, kThreads, L::bytes, stream>>>(a);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dk(const ChunkArgs &a, cudaStream_t stream) {
  if (a.bf16)
    return a.per_channel ? launch_t<DK, true, true>(a, stream) : launch_t<DK, true, false>(a, stream);
  return a.per_channel ? launch_t<DK, false, true>(a, stream) : launch_t<DK, false, false>(a, stream);
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream) {
  switch (a.dk) {
    case 32: return launch_dk<32>(a, stream);
    case 64: return launch_dk<64>(a, stream);
    case 128: return launch_dk<128>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdr
