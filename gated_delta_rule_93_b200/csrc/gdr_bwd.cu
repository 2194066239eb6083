// Backward of the gated delta-rule recurrence on CUDA cores (fp32): the
// gradients of q, k, v, g = log alpha, beta and S0 from dL/do and dL/dS_T.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5
// (backpropagation through the recurrence, with recomputation).  One step
// and its reverse, per (b, h), with S' = S_{t-1} Diag(alpha_t):
//     p = S' k,  u = beta (v - p),  S_t = S' + u k^T,  o_t = S_t q
//     G += do q^T;  dq = S_t^T do;  du = G k;  dbeta = du . (v - p)
//     dv = beta du;  dp = -beta du;  dk = G^T u + S'^T dp
//     dS' = G + dp k^T;  dg_j = sum_i S'[i][j] dS'[i][j];  G <- dS' Diag(alpha)
// (G = dL/dS_t; dS0 = G after the first step).
//
// One CTA per (b, h), 16 warps.  Rows of the state are independent in the
// recurrence: warp w owns rows w, w + 16, ... and lane l the key channels
// l, l + 32, ..., so S and G stay in registers (32 floats each at d = 128)
// and a row's dot products are warp reductions.  The sums over rows (dq, dk,
// dg, dbeta) go through shared memory once per token.
// Recomputation: a forward sweep stores the state at every 8th token
// (checkpoints); then, 8 tokens at a time from the last, the states are
// recomputed from their checkpoint into a stash and walked in reverse.
// Both live in the caller's workspace, element-major ([element][thread], so
// a warp's access is one contiguous 128-byte line; each thread reads back
// only what it wrote); a stash holds 8 states of 64 KB at d = 128, each read
// back within 8 tokens of being written.  The token vectors of a 64-token
// chunk (k, q, v, g, beta, dL/do) are staged in shared memory as fp32 by
// the whole CTA with coalesced loads before the chunk is processed.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 64;  // tokens staged in shared memory at a time
constexpr int kSub = 8;     // tokens per checkpoint / stash

struct BwdArgs {
  const void *q, *k, *v;
  const float *g, *beta, *S0, *dout, *dST;
  float *dq, *dk, *dv, *dg, *dbeta, *dS0;
  float *ws;
  int B, T, H, d, bf16, per_channel;
};

__device__ __forceinline__ float ld_in(const void *p, size_t i, int bf16) {
  if (bf16) {
    const uint16_t u = reinterpret_cast<const uint16_t *>(p)[i];
    return __uint_as_float((uint32_t)u << 16);
  }
  return reinterpret_cast<const float *>(p)[i];
}

template <int RW>
__device__ __forceinline__ void warp_sum_rows(float (&x)[RW]) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int r = 0; r < RW; ++r) x[r] += __shfl_xor_sync(0xffffffffu, x[r], off);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// NC = d / 32 key channels per lane, RW = d / 16 rows per warp.
template <int NC, int RW>
__global__ void __launch_bounds__(kThreads, 1) gdr_bwd_kernel(BwdArgs a) {
  constexpr int D = NC * 32;
  constexpr int E = NC * RW;  // state elements per thread
  // shared memory: per-warp partial sums [2][kWarps][3 D + 1], then the
  // staged chunk: k, q, v, dL/do [kChunk][D], g [kChunk][D or 1], beta [kChunk]
  extern __shared__ float smem[];
  float(*red)[kWarps][3 * D + 1] = reinterpret_cast<float(*)[kWarps][3 * D + 1]>(smem);
  float *sk = smem + 2 * kWarps * (3 * D + 1);
  float *sq = sk + kChunk * D, *sv = sq + kChunk * D, *sdo = sv + kChunk * D;
  float *sg = sdo + kChunk * D;
  float *sb = sg + kChunk * (a.per_channel ? D : 1);
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int T = a.T, H = a.H;
  const int nsub = (T + kSub - 1) / kSub;
  const int nch = (T + kChunk - 1) / kChunk;
  const size_t SS = (size_t)D * D;
  float *ckpt = a.ws + (size_t)bh * (nsub + 1 + kSub) * SS;  // [nsub + 1][E][thread]
  float *stash = ckpt + (size_t)(nsub + 1) * SS;              // [kSub][E][thread]
  auto at = [&](float *base, int slot) { return base + (size_t)slot * SS + tid; };
  auto sidx = [&](int r, int c) { return (size_t)(w + 16 * r) * D + l + 32 * c; };

  float S[RW][NC], G[RW][NC];
  {
    const float *s0 = a.S0 ? a.S0 + (size_t)bh * SS : nullptr;
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) S[r][c] = s0 ? s0[sidx(r, c)] : 0.f;
  }

  // tokens [t0, t1) of this (b, h) into shared memory (all threads;
  // bracketed by barriers)
  auto stage = [&](int t0, int t1, bool with_q, bool with_do) {
    __syncthreads();  // the previous chunk's reads are done
    const int n = (t1 - t0) * D;
    for (int i = tid; i < n; i += kThreads) {
      const int t = i / D, j = i - t * D;
      const size_t x = (((size_t)b * T + t0 + t) * H + h) * D + j;
      sk[i] = ld_in(a.k, x, a.bf16);
      sv[i] = ld_in(a.v, x, a.bf16);
      if (with_q) sq[i] = ld_in(a.q, x, a.bf16);
      if (with_do) sdo[i] = a.dout[x];
      if (a.per_channel) sg[i] = a.g[x];
    }
    for (int t = tid; t < t1 - t0; t += kThreads) {
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      if (!a.per_channel) sg[t] = a.g[tok];
      sb[t] = a.beta[tok];
    }
    __syncthreads();
  };
  // per-token inputs of this thread: k, q, alpha at its channels, v at its
  // rows (token tl of the staged chunk)
  float kk[NC], qq[NC], al[NC], vv[RW], be;
  auto load = [&](int tl) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      kk[c] = sk[tl * D + l + 32 * c];
      qq[c] = sq[tl * D + l + 32 * c];
      al[c] = __expf(a.per_channel ? sg[tl * D + l + 32 * c] : sg[tl]);
    }
#pragma unroll
    for (int r = 0; r < RW; ++r) vv[r] = sv[tl * D + w + 16 * r];
    be = sb[tl];
  };
  // one forward step in place: S <- S Diag(alpha) + u k^T; returns nothing
  auto step = [&](float (&X)[RW][NC]) {
    float p[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        X[r][c] *= al[c];
        acc = fmaf(X[r][c], kk[c], acc);
      }
      p[r] = acc;
    }
    warp_sum_rows<RW>(p);
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const float u = be * (vv[r] - p[r]);
#pragma unroll
      for (int c = 0; c < NC; ++c) X[r][c] = fmaf(u, kk[c], X[r][c]);
    }
  };
  auto store = [&](float *dst, const float (&X)[RW][NC]) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) dst[(r * NC + c) * kThreads] = X[r][c];
  };
  auto fetch = [&](const float *src, float (&X)[RW][NC]) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) X[r][c] = src[(r * NC + c) * kThreads];
  };

  // ---- forward sweep: checkpoints at every kSub-th token
  for (int ch = 0; ch < nch; ++ch) {
    const int t0 = ch * kChunk, t1 = min(T, t0 + kChunk);
    stage(t0, t1, false, false);
    for (int t = t0; t < t1; ++t) {
      if (t % kSub == 0) store(at(ckpt, t / kSub), S);
      load(t - t0);
      step(S);
    }
  }

  // ---- reverse: G = dL/dS_T
  {
    const float *d = a.dST ? a.dST + (size_t)bh * SS : nullptr;
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) G[r][c] = d ? d[sidx(r, c)] : 0.f;
  }
  for (int ch = nch - 1; ch >= 0; --ch) {
    const int c0 = ch * kChunk, c1 = min(T, c0 + kChunk);
    stage(c0, c1, true, true);
    for (int t0 = c0 + ((c1 - 1 - c0) / kSub) * kSub; t0 >= c0; t0 -= kSub) {
    const int t1 = min(c1, t0 + kSub);
    fetch(at(ckpt, t0 / kSub), S);
    for (int t = t0; t < t1; ++t) {  // the states S_{t-1} into the stash
      store(at(stash, t - t0), S);
      load(t - c0);
      step(S);
    }
    for (int t = t1 - 1; t >= t0; --t) {
      load(t - c0);
      const size_t tok = ((size_t)b * T + t) * H + h;
      float Sp[RW][NC];
      fetch(at(stash, t - t0), Sp);
      float p[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          Sp[r][c] *= al[c];
          acc = fmaf(Sp[r][c], kk[c], acc);
        }
        p[r] = acc;
      }
      warp_sum_rows<RW>(p);
      float u[RW], dO[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        u[r] = be * (vv[r] - p[r]);
        dO[r] = sdo[(t - c0) * D + w + 16 * r];
      }
      // dq = S_t^T do (partial over this warp's rows); G += do q^T
      float dqp[NC], dkp[NC], dgp[NC];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          acc = fmaf(fmaf(u[r], kk[c], Sp[r][c]), dO[r], acc);
          G[r][c] = fmaf(dO[r], qq[c], G[r][c]);
        }
        dqp[c] = acc;
      }
      // du = G k
      float du[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) acc = fmaf(G[r][c], kk[c], acc);
        du[r] = acc;
      }
      warp_sum_rows<RW>(du);
      float dbp = 0.f;
#pragma unroll
      for (int r = 0; r < RW; ++r) dbp = fmaf(du[r], vv[r] - p[r], dbp);
      if (l < RW) {  // lane r writes row r's dv (every lane holds every du)
        float x = 0.f;
#pragma unroll
        for (int r = 0; r < RW; ++r) x = (l == r) ? du[r] : x;
        a.dv[tok * D + w + 16 * l] = be * x;
      }
      // dk = G^T u + S'^T dp;  dS' = G + dp k^T;  dg = diag(S'^T dS');  G <- dS' Diag(alpha)
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        float ak = 0.f, ag = 0.f;
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          const float dp = -be * du[r];
          ak = fmaf(G[r][c], u[r], ak);
          ak = fmaf(Sp[r][c], dp, ak);
          const float dsp = fmaf(dp, kk[c], G[r][c]);
          ag = fmaf(Sp[r][c], dsp, ag);
          G[r][c] = dsp * al[c];
        }
        dkp[c] = ak;
        dgp[c] = ag;
      }
      // sums over the 16 warps' rows
      float *rb = &red[t & 1][w][0];
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        rb[l + 32 * c] = dqp[c];
        rb[D + l + 32 * c] = dkp[c];
        rb[2 * D + l + 32 * c] = dgp[c];
      }
      if (l == 0) rb[3 * D] = dbp;
      __syncthreads();
      for (int i = tid; i < 3 * D + 1; i += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) s += red[t & 1][ww][i];
        if (i < D)
          a.dq[tok * D + i] = s;
        else if (i < 2 * D)
          a.dk[tok * D + i - D] = s;
        else if (i < 3 * D) {
          if (a.per_channel) a.dg[tok * D + i - 2 * D] = s;
        } else {
          a.dbeta[tok] = s;
        }
      }
      if (!a.per_channel) {  // scalar gate: dg = sum over channels of dg_j
        // (the per-channel sums are in red[t & 1][*][2D ..); warp 0 adds them)
        if (w == 0) {
          float s = 0.f;
          for (int i = l; i < D; i += 32)
            for (int ww = 0; ww < kWarps; ++ww) s += red[t & 1][ww][2 * D + i];
          s = warp_sum(s);
          if (l == 0) a.dg[tok] = s;
        }
      }
    }
    }
  }
  if (a.dS0) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int c = 0; c < NC; ++c) a.dS0[(size_t)bh * SS + sidx(r, c)] = G[r][c];
  }
}

}  // namespace

size_t bwd_ws_bytes(int B, int T, int H, int d) {
  if (B <= 0 || H <= 0 || T < 0) return 0;
  const size_t nsub = (size_t)(T + kSub - 1) / kSub;
  return (size_t)B * H * (nsub + 1 + kSub) * (size_t)d * d * sizeof(float);
}

cudaError_t launch_bwd(const void *q, const void *k, const void *v, int bf16, const float *g,
                       int per_channel, const float *beta, const float *S0, const float *dout,
                       const float *dST, float *dq, float *dk, float *dv, float *dg,
                       float *dbeta, float *dS0, int B, int T, int H, int d, void *ws,
                       cudaStream_t stream) {
  BwdArgs a{q, k, v, g, beta, S0, dout, dST, dq, dk, dv, dg, dbeta, dS0,
            static_cast<float *>(ws), B, T, H, d, bf16, per_channel};
  const unsigned grid = (unsigned)((size_t)B * H);
  const size_t smem = (2 * kWarps * (3 * (size_t)d + 1) + 4 * (size_t)kChunk * d +
                      (size_t)kChunk * (per_channel ? d : 1) + kChunk) *
                     sizeof(float);
  auto go = [&](auto kern) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
  };
  switch (d) {
    case 32: return go(gdr_bwd_kernel<1, 2>);
    case 64: return go(gdr_bwd_kernel<2, 4>);
    case 128: return go(gdr_bwd_kernel<4, 8>);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdr
