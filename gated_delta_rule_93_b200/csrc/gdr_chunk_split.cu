// Chunkwise gated delta-rule forward on the sm_100a tensor cores for the
// shapes the warp-specialised bf16 kernel does not take: fp32 inputs, and
// head dims d_k, d_v in {32, 64, 128} other than bf16 with d_k = d_v = 128.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5
// (inter-chunk state recursion, intra-chunk output, log-space gates) and the
// WY/UT form of the delta rule from "Linear Attention Variants (RetNet, GLA,
// DeltaNet, Based)", DeltaNet section.  In the state's own orientation (S is
// d_v x d_k, one TMEM lane per value channel i) and for one chunk of C = 64
// tokens, with gc_r the cumulative log decay from the chunk start and m a
// per-key-channel reference (gc at row 31 for a per-channel gate, 0 for a
// scalar gate):
//
//   K~ = K e^{gc - m},  Q~ = Q e^{gc - m},  K^ = K e^{m - gc}
//   D1  = [K~; Q~] K^^T                   (tcgen05, M = 128, N = 64)
//   A   = strict_tril(beta_r D1_KK Gamma),  P = tril_incl(D1_QK Gamma)
//         (Gamma_rs = e^{gc_r - gc_s} for a scalar gate, 1 per channel)
//   [Z | O_a] = S' [K~; Q~]^T,  S' = S Diag(e^{m})     (tcgen05, A = S' in TMEM)
//   T   = (I + A)^{-1} Diag(beta)         (forward substitution, fp32)
//   U^T = (V^T - zf Z) T^T                 (zf_r = e^{gc_r} scalar gate, 1 per channel)
//   O^T = zf O_a + U^T P^T
//   S   = S Diag(e^{gc_last}) + U^T (K e^{gc_last - gc})
//
// Every operand is carried as two bf16 terms, x = hi + lo with
// |x - hi - lo| <= 2^-18 |x|, and each product as three bf16 MMAs (hi hi,
// hi lo, lo hi) into one fp32 accumulator, so the contractions keep close to
// fp32 accuracy (the dropped lo lo term and the split are below 2^-16
// relative) on the bf16 tensor-core path.  The state stays fp32 in TMEM;
// T is solved in fp32 on the CUDA cores.
//
// A per-channel gate's factors e^{+-(gc - m)} are bounded by 2^100 (the lo
// terms of the split stay normal numbers); a chunk whose decay within 32
// tokens exceeds that has those factors zeroed and sets the range bit of the
// status word, so the call reports GDR_ERR_RANGE instead of a wrong result.
// The scalar gate's factors are pairwise and never exceed 1.
//
// The same file holds the chunked DPLR transition (below), built the same
// way.
//
// One CTA per (b, h), 128 threads, sequential phases (load and split ->
// D1, Z, O_a -> A, P, U's right-hand side, decay of S -> T -> U -> O_b and
// the state update -> output), each MMA group waited on with a bounded
// mbarrier wait.  d_k = 32 is zero-padded to 64 on chip; d_v < 128 leaves
// the upper TMEM lanes at zero.  A ragged last chunk is zero-padded
// (k = q = v = 0, beta = 0, g = 0), which leaves the state untouched; its
// padded output rows are not stored.
#include "gdr_internal.cuh"
#include "gdr_tc_util.cuh"

namespace gdr {
namespace {

using namespace sm100;
using namespace tcu;

constexpr int C = 64;
constexpr int kThreadsD = 256;  // both kernels: 8 warps, two per TMEM lane quarter
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kMaxExp = 100.f * kLn2;  // largest |gc - m| of a scaled factor

// Shared memory (bytes from a 1024-byte aligned base).  bf16 tiles in the
// 128-byte swizzle, K-major, 64 columns per block:
//   KQ    [K~; Q~] 128 rows x DK (hi, lo)
//   KH    K^ 64 rows x DK (hi, lo); after D1: A in fp32 [64][64]
//   KB    (K e^{gl - gc})^T  DK rows x 64 (hi, lo)
//   TT, PP  T and P 64 x 64 (hi, lo)
//   GC    per-channel cumulative log decays [64][DK] fp32
template <int DK>
struct Layout {
  static constexpr uint32_t kKQBlk = 128 * 128, kKHBlk = 64 * 128;
  static constexpr uint32_t KQ_HI = 0, KQ_LO = KQ_HI + (DK / 64) * kKQBlk;
  static constexpr uint32_t KH_HI = KQ_LO + (DK / 64) * kKQBlk,
                            KH_LO = KH_HI + (DK / 64) * kKHBlk;
  static constexpr uint32_t KB_HI = KH_LO + (DK / 64) * kKHBlk, KB_LO = KB_HI + DK * 128;
  static constexpr uint32_t TT_HI = KB_LO + DK * 128, TT_LO = TT_HI + 8192;
  static constexpr uint32_t PP_HI = TT_LO + 8192, PP_LO = PP_HI + 8192;
  static constexpr uint32_t GC = PP_LO + 8192;
  static constexpr uint32_t VEC = GC + 64 * DK * 4;  // 768 floats
  static constexpr uint32_t BAR = VEC + 768 * 4, MISC = BAR + 16, END = MISC + 16;
  static constexpr size_t bytes = END + 1024;
  static_assert(2 * (DK / 64) * kKHBlk >= 64 * 64 * 4, "A overlays K^");
  static_assert(bytes <= 232448, "shared memory budget");
};

// TMEM columns: S fp32 [DK], S' hi / lo as bf16 pairs [DK/2 each], D1 (then
// O_b) [64], Z (then U's right-hand side, hi | lo) and O_a [128], U [64].
template <int DK>
struct Cols {
  static constexpr uint32_t S = 0, SH = DK, SL = DK + DK / 2, D1 = 2 * DK, ZO = 2 * DK + 64,
                            U = 2 * DK + 192;
  static_assert(U + 64 <= 512, "TMEM columns");
};

// 8 consecutive input elements (fp32 if !BF, else bf16) of a [B, T, H, d]
// tensor at element offset `off`.  Callers pass an in-range offset for
// every lane (a clamped one where the element is padding) and select zero
// afterwards, so that the loads carry no branch and all of a phase's loads
// can be in flight together.
template <bool BF>
__device__ __forceinline__ void ld8(const void *p, size_t off, float (&x)[8]) {
  if (BF) {
    const uint4 u = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p) +
                                                     off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16(w[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  } else {
    const float4 *q = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p) + off);
    const float4 a = q[0], b = q[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
}

template <bool BF>
__device__ __forceinline__ float ld1(const void *p, size_t off) {
  if (BF) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[off]);
  return reinterpret_cast<const float *>(p)[off];
}

template <bool BF>
__device__ __forceinline__ void st1(void *p, size_t off, float x) {
  if (BF)
    reinterpret_cast<__nv_bfloat16 *>(p)[off] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float *>(p)[off] = x;
}

// Element (row r, column c0) of a chunk's [64][d] input block starting at
// token row offset `tok0` (token stride H): the offset of the element when
// it exists (r < L, c0 < d), else of the chunk's first element.
__device__ __forceinline__ size_t in_off(size_t tok0, int r, int c0, int H, int d, bool valid) {
  return valid ? (tok0 + (size_t)r * H) * d + c0 : tok0 * d;
}

// 16 consecutive fp32 of row r of a swizzled [64][16 float4] matrix,
// columns 16 q .. 16 q + 15.
__device__ __forceinline__ void ld_row16(const float4 *N4, int r, int q, float (&x)[16]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float4 v = N4[r * 16 + ((4 * q + u) ^ (r & 15))];
    x[4 * u] = v.x;
    x[4 * u + 1] = v.y;
    x[4 * u + 2] = v.z;
    x[4 * u + 3] = v.w;
  }
}

// X = (I + s N)^{-1} for a strictly lower-triangular 64 x 64 N (s = +1 or
// -1), by 16 x 16 blocks; threads 0-63 (the other warps do not take part;
// 64-thread named barrier 1).  N is fp32 [64][16 float4] with float4 k of
// row r at k ^ (r % 16); X goes to Y [64][64] fp32 ([row][column]: a warp's
// lanes hit distinct banks).  With L = I + s N:
//   X_ii = L_ii^{-1}   (four blocks at once, one column per thread, by
//                       forward substitution)
//   X_ij = -s X_ii sum_{k=j}^{i-1} N_ik X_kj   (i > j, in three levels
//                       i - j = 1, 2, 3; 48, 32, then 16 threads, one column
//                       each)
// The products' loops stay rolled over blocks, so the code is small: a
// fully unrolled 64-row substitution is ~40 KB of straight-line code and
// ran from instruction-cache misses.
template <int S>
__device__ __forceinline__ void block_solve(const float4 *N4, float *Y, int t) {
  {  // diagonal blocks: block i = t / 16, column c = 16 i + t % 16
    const int i = t >> 4, cc = t & 15, c = 16 * i + cc;
    float y[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float nr[16];
      ld_row16(N4, 16 * i + k, i, nr);
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < k; ++j) sum = fmaf(nr[j], y[j], sum);
      y[k] = (k == cc ? 1.f : 0.f) - (float)S * sum;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) Y[(16 * i + k) * 64 + c] = y[k];
#pragma unroll 1
    for (int r = 0; r < 16 * i; ++r) Y[r * 64 + c] = 0.f;  // above the diagonal blocks
  }
  asm volatile("bar.sync 1, 64;" ::: "memory");
#pragma unroll 1
  for (int lvl = 1; lvl < 4; ++lvl) {
    if (t < 16 * (4 - lvl)) {
      const int j = t >> 4, i = j + lvl, c = 16 * j + (t & 15);
      float m[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) m[u] = 0.f;
#pragma unroll 1
      for (int k = j; k < i; ++k) {  // m += N_ik X_kj[:, c], four rows of N_ik at a time
        float xk[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) xk[p] = Y[(16 * k + p) * 64 + c];
#pragma unroll
        for (int ug = 0; ug < 4; ++ug) {
          float n0[16], n1[16], n2[16], n3[16];
          ld_row16(N4, 16 * i + 4 * ug + 0, k, n0);
          ld_row16(N4, 16 * i + 4 * ug + 1, k, n1);
          ld_row16(N4, 16 * i + 4 * ug + 2, k, n2);
          ld_row16(N4, 16 * i + 4 * ug + 3, k, n3);
#pragma unroll
          for (int p = 0; p < 16; ++p) {  // four independent chains, interleaved
            m[4 * ug + 0] = fmaf(n0[p], xk[p], m[4 * ug + 0]);
            m[4 * ug + 1] = fmaf(n1[p], xk[p], m[4 * ug + 1]);
            m[4 * ug + 2] = fmaf(n2[p], xk[p], m[4 * ug + 2]);
            m[4 * ug + 3] = fmaf(n3[p], xk[p], m[4 * ug + 3]);
          }
        }
      }
#pragma unroll
      for (int ug = 0; ug < 4; ++ug) {  // X_ij[:, c] = -s X_ii m, four rows at a time
        float x0[16], x1[16], x2[16], x3[16];
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const float4 *r0 = reinterpret_cast<const float4 *>(Y + (16 * i + 4 * ug + 0) * 64 + 16 * i);
        const float4 *r1 = reinterpret_cast<const float4 *>(Y + (16 * i + 4 * ug + 1) * 64 + 16 * i);
        const float4 *r2 = reinterpret_cast<const float4 *>(Y + (16 * i + 4 * ug + 2) * 64 + 16 * i);
        const float4 *r3 = reinterpret_cast<const float4 *>(Y + (16 * i + 4 * ug + 3) * 64 + 16 * i);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 v0 = r0[q], v1 = r1[q], v2 = r2[q], v3 = r3[q];
          x0[4 * q] = v0.x; x0[4 * q + 1] = v0.y; x0[4 * q + 2] = v0.z; x0[4 * q + 3] = v0.w;
          x1[4 * q] = v1.x; x1[4 * q + 1] = v1.y; x1[4 * q + 2] = v1.z; x1[4 * q + 3] = v1.w;
          x2[4 * q] = v2.x; x2[4 * q + 1] = v2.y; x2[4 * q + 2] = v2.z; x2[4 * q + 3] = v2.w;
          x3[4 * q] = v3.x; x3[4 * q + 1] = v3.y; x3[4 * q + 2] = v3.z; x3[4 * q + 3] = v3.w;
        }
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          a0 = fmaf(x0[p], m[p], a0);
          a1 = fmaf(x1[p], m[p], a1);
          a2 = fmaf(x2[p], m[p], a2);
          a3 = fmaf(x3[p], m[p], a3);
        }
        Y[(16 * i + 4 * ug + 0) * 64 + c] = -(float)S * a0;
        Y[(16 * i + 4 * ug + 1) * 64 + c] = -(float)S * a1;
        Y[(16 * i + 4 * ug + 2) * 64 + c] = -(float)S * a2;
        Y[(16 * i + 4 * ug + 3) * 64 + c] = -(float)S * a3;
      }
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
  }
}

// hi / lo bf16 of 8 values into the 16-byte chunk at `off` of two tiles.
__device__ __forceinline__ void put8(uint8_t *hi_tile, uint8_t *lo_tile, uint32_t off,
                                     const float (&x)[8]) {
  float h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) split_bf16(x[e], h[e], l[e]);
  *reinterpret_cast<uint4 *>(hi_tile + off) =
      make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]),
                 pack_bf16(h[6], h[7]));
  *reinterpret_cast<uint4 *>(lo_tile + off) =
      make_uint4(pack_bf16(l[0], l[1]), pack_bf16(l[2], l[3]), pack_bf16(l[4], l[5]),
                 pack_bf16(l[6], l[7]));
}

// 32 fp32 values as hi / lo bf16 pairs: 16 TMEM columns each at th and tl.
__device__ __forceinline__ void tmem_put_split32(uint32_t th, uint32_t tl, const float (&x)[32]) {
  uint32_t hu[16], lu[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float h0, l0, h1, l1;
    split_bf16(x[2 * e], h0, l0);
    split_bf16(x[2 * e + 1], h1, l1);
    hu[e] = pack_bf16(h0, h1);
    lu[e] = pack_bf16(l0, l1);
  }
  tmem_st16u(th, hu);
  tmem_st16u(tl, lu);
}

__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, bool ok) {
  ok = ok && mbar_wait_bounded(bar, parity, kWaitNs);
  return __syncthreads_and(ok) != 0;
}

// Generic shared-memory and TMEM writes of every thread -> the next MMA.
__device__ __forceinline__ void sync_for_mma() {
  fence_proxy_async_smem();
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// Prologue maps (raw projections in): "Decoding Hybrid Linear Attention
// Architectures", section 4 (beta in (0, 1), alpha in (0, 1], gates in log
// space) and section 3 item 2 (the erase is a projector along a unit key):
// beta = sigmoid(b), g = -s_h softplus(a), q, k <- x / sqrt(|x|^2 + eps).
constexpr float kNormEps = 1e-6f;
__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }

// beta of rows lane, lane + 32 (one warp); from logits when `logit`.
__device__ __forceinline__ void load_beta(float *betav, const float *beta, size_t tok0, int H,
                                          int L, int lane, bool logit) {
  float b0 = lane < L ? beta[tok0 + (size_t)lane * H] : 0.f;
  float b1 = lane + 32 < L ? beta[tok0 + (size_t)(lane + 32) * H] : 0.f;
  if (logit) {
    b0 = lane < L ? sigmoid_f(b0) : 0.f;
    b1 = lane + 32 < L ? sigmoid_f(b1) : 0.f;
  }
  betav[lane] = b0;
  betav[lane + 32] = b1;
}

// 1 / sqrt(|x|^2 + eps) of row r of k (flags & 2) and q (flags & 1); this
// thread holds the columns [hf DK/4, hf DK/4 + DK/4) and the three threads
// beside it (thread ^ 1, ^ 2, ^ 3) the others, so the sums meet with two
// shuffles.  Every lane of the warp calls this.
template <bool BF, int DK>
__device__ __forceinline__ void row_inv_norms(const void *k, const void *q, size_t tok0, int r,
                                              int hf, int H, int dk, int L, int flags, float &rk,
                                              float &rq) {
  float sk = 0.f, sq = 0.f;
#pragma unroll
  for (int g8 = 0; g8 < DK / 32; ++g8) {
    const int c0 = hf * (DK / 4) + 8 * g8;
    const bool valid = r < L && c0 < dk;
    const size_t off = in_off(tok0, r, c0, H, dk, valid);
    float kx[8], qx[8];
    ld8<BF>(k, off, kx);
    ld8<BF>(q, off, qx);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sk = fmaf(valid ? kx[e] : 0.f, valid ? kx[e] : 0.f, sk);
      sq = fmaf(valid ? qx[e] : 0.f, valid ? qx[e] : 0.f, sq);
    }
  }
  sk += __shfl_xor_sync(0xffffffffu, sk, 1);
  sq += __shfl_xor_sync(0xffffffffu, sq, 1);
  sk += __shfl_xor_sync(0xffffffffu, sk, 2);
  sq += __shfl_xor_sync(0xffffffffu, sq, 2);
  rk = (flags & 2) ? rsqrtf(sk + kNormEps) : 1.f;
  rq = (flags & 1) ? rsqrtf(sq + kNormEps) : 1.f;
}

template <int DK, bool PC, bool BF>
__global__ void __launch_bounds__(kThreadsD, 1) gdr_chunk_split_kernel(ChunkArgs a) {
  using LY = Layout<DK>;
  using TC = Cols<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  // 8 warps: warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 (value
  // channels) and split each per-lane phase's columns or rows between them (hs)
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, lq = warp & 3, hs = warp >> 2;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H, H = a.H;
  const int dk = a.dk, dv = a.dv;
  // sequence b: token rows [seq0, seq0 + Tb) of the [B, T] (or packed [1, total]) layout
  // (packed: cu_seqlens clamped into [0, total] and non-decreasing)
  const int seq0 = a.cu_seqlens ? min(max(a.cu_seqlens[b], 0), a.T) : b * a.T;
  const int Tb = a.cu_seqlens ? min(max(a.cu_seqlens[b + 1], seq0), a.T) - seq0 : a.T;
  const int n = (Tb + C - 1) / C;
  const bool add = a.additive != 0, pro = a.prologue != 0;
  const float gsc = pro ? a.gate_scale[h] : 0.f;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + LY::BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + LY::MISC);
  float *vec = reinterpret_cast<float *>(sm + LY::VEC);
  float *gcs = vec;          // [64] scalar gate: cumulative log decay
  float *zf = vec + 64;      // [64] e^{gc_r} (scalar gate) or 1
  float *ebar = vec + 128;   // [64] scalar gate: e^{gl - gc_r}
  float *betav = vec + 192;  // [64]
  float *mref = vec + 256;   // [128] per channel: m_j
  float *em = vec + 384;     // [128] per channel: e^{m_j}
  float *egl = vec + 512;    // [128] e^{gl_j} (scalar gate: every entry e^{gl})
  float *glv = vec + 640;    // [128] per channel: gl_j
  float *gcm = reinterpret_cast<float *>(sm + LY::GC);  // [64][DK]
  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  const uint32_t lb = tm + ((uint32_t)(lq * 32) << 16);  // this warp's lanes
  const int i = lq * 32 + lane;                          // value channel (TMEM lane)

  // S = S0 (or 0); lanes >= d_v and columns >= d_k stay 0
#pragma unroll 1
  for (int q = hs; q < DK / 32; q += 2) {
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = 32 * q + e;
      x[e] = (a.S0 && i < dv && j < dk) ? a.S0[((size_t)bh * dv + i) * dk + j] : 0.f;
    }
    tmem_st32(lb + TC::S + 32 * q, x);
  }
  tmem_wait_st();

  constexpr uint32_t ID_D1 = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_ZO = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t ID_64 = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_S = idesc_bf16(128, DK, 0, 0);
  const uint32_t s_kqh = smem_u32(sm + LY::KQ_HI), s_kql = smem_u32(sm + LY::KQ_LO);
  const uint32_t s_khh = smem_u32(sm + LY::KH_HI), s_khl = smem_u32(sm + LY::KH_LO);
  const uint32_t s_kbh = smem_u32(sm + LY::KB_HI), s_kbl = smem_u32(sm + LY::KB_LO);
  const uint32_t s_tth = smem_u32(sm + LY::TT_HI), s_ttl = smem_u32(sm + LY::TT_LO);
  const uint32_t s_pph = smem_u32(sm + LY::PP_HI), s_ppl = smem_u32(sm + LY::PP_LO);
  float4 *Af4 = reinterpret_cast<float4 *>(sm + LY::KH_HI);  // A [64][16 float4], swizzled

  uint32_t ph = 0;
  bool ok = true;
  auto mma_wait = [&]() {
    if (t == 0) mma_commit(bar);
    ok = wait_all(bar, ph, ok);
    ph ^= 1;
    tc_fence_after();
  };

#pragma unroll 1
  for (int c = 0; c < n && ok; ++c) {
    const int t0 = c * C, L = min(C, Tb - t0);
    const size_t tok0 = ((size_t)seq0 + t0) * H + h;  // token index of row 0
    // ---- gates
    if (PC) {
      if (t < DK) {
        const int j = t;
        float acc = 0.f, m = 0.f;
#pragma unroll 8
        for (int r = 0; r < C; ++r) {
          const float x = (r < L && j < dk) ? a.g[(tok0 + (size_t)r * H) * dk + j] : 0.f;
          acc += pro ? ((r < L && j < dk) ? -gsc * softplus_f(x) : 0.f) : x;
          gcm[r * DK + j] = acc;
          if (r == 31) m = acc;
        }
        mref[j] = m;
        em[j] = __expf(m);
        egl[j] = __expf(acc);
        glv[j] = acc;
      }
      if (warp == 3 && !add) load_beta(betav, a.beta, tok0, H, L, lane, pro);
      if (t < 64) zf[t] = 1.f;
    } else {
      if (warp == 0) {
        float x0 = lane < L ? a.g[tok0 + (size_t)lane * H] : 0.f;
        float x1 = lane + 32 < L ? a.g[tok0 + (size_t)(lane + 32) * H] : 0.f;
        if (pro) {  // logits -> g = -s_h softplus(a)
          x0 = lane < L ? -gsc * softplus_f(x0) : 0.f;
          x1 = lane + 32 < L ? -gsc * softplus_f(x1) : 0.f;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
          if (lane >= off) {
            x0 += y0;
            x1 += y1;
          }
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const float gl = __shfl_sync(0xffffffffu, x1, 31);
        gcs[lane] = x0;
        gcs[lane + 32] = x1;
        zf[lane] = __expf(x0);
        zf[lane + 32] = __expf(x1);
        ebar[lane] = __expf(gl - x0);
        ebar[lane + 32] = __expf(gl - x1);
#pragma unroll
        for (int e = 0; e < 4; ++e) egl[lane + 32 * e] = __expf(gl);
      }
      if (warp == 1 && !add) load_beta(betav, a.beta, tok0, H, L, lane, pro);
    }
    __syncthreads();
    // ---- S' = S Diag(e^{m}) as hi / lo bf16 in TMEM
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TC::S + 32 * q, x);
      uint32_t hu[16], lu[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float f0 = PC ? em[32 * q + 2 * e] : 1.f, f1 = PC ? em[32 * q + 2 * e + 1] : 1.f;
        float h0, l0, h1, l1;
        split_bf16(x[2 * e] * f0, h0, l0);
        split_bf16(x[2 * e + 1] * f1, h1, l1);
        hu[e] = pack_bf16(h0, h1);
        lu[e] = pack_bf16(l0, l1);
      }
      tmem_st16u(lb + TC::SH + 16 * q, hu);
      tmem_st16u(lb + TC::SL + 16 * q, lu);
    }
    // ---- K~, Q~, K^, (K e^{gl - gc})^T tiles: row r = t / 4, quarter t % 4 of the columns
    {
      const int r = t >> 2, hf = t & 3;
      bool range_bad = false;
      float rk = 1.f, rq = 1.f;  // prologue: 1 / |k_r|, 1 / |q_r| (threads 4 r .. 4 r + 3 hold the row)
      if (pro && a.norm_qk) row_inv_norms<BF, DK>(a.k, a.q, tok0, r, hf, H, dk, L, a.norm_qk, rk, rq);
#pragma unroll
      for (int g8 = 0; g8 < DK / 32; ++g8) {
        const int c0 = hf * (DK / 4) + 8 * g8;
        const bool valid = r < L && c0 < dk;
        const size_t off = in_off(tok0, r, c0, H, dk, valid);
        float kx[8], qx[8];
        ld8<BF>(a.k, off, kx);
        ld8<BF>(a.q, off, qx);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          kx[e] = valid ? kx[e] * rk : 0.f;
          qx[e] = valid ? qx[e] * rq : 0.f;
        }
        float kt[8], qt[8], kh[8], kb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = c0 + e;
          if (PC) {
            const float x = gcm[r * DK + j] - mref[j];
            const bool inr = fabsf(x) <= kMaxExp;
            range_bad |= !inr && (kx[e] != 0.f || qx[e] != 0.f);
            const float up = inr ? __expf(x) : 0.f, dn = inr ? __expf(-x) : 0.f;
            kt[e] = kx[e] * up;
            qt[e] = qx[e] * up;
            kh[e] = kx[e] * dn;
            kb[e] = kx[e] * __expf(glv[j] - gcm[r * DK + j]);
          } else {
            kt[e] = kx[e];
            qt[e] = qx[e];
            kh[e] = kx[e];
            kb[e] = kx[e] * ebar[r];
          }
        }
        const uint32_t blk = (uint32_t)(c0 >> 6), cc = (uint32_t)(c0 & 63);
        put8(sm + LY::KQ_HI + blk * LY::kKQBlk, sm + LY::KQ_LO + blk * LY::kKQBlk,
             sw128_off(r, cc), kt);
        put8(sm + LY::KQ_HI + blk * LY::kKQBlk, sm + LY::KQ_LO + blk * LY::kKQBlk,
             sw128_off(64 + r, cc), qt);
        put8(sm + LY::KH_HI + blk * LY::kKHBlk, sm + LY::KH_LO + blk * LY::kKHBlk,
             sw128_off(r, cc), kh);
#pragma unroll
        for (int e = 0; e < 8; ++e) {  // transposed: row j, column r
          float hi, lo;
          split_bf16(kb[e], hi, lo);
          const uint32_t off = sw128_off(c0 + e, r);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::KB_HI + off) = __float2bfloat16_rn(hi);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::KB_LO + off) = __float2bfloat16_rn(lo);
        }
      }
      if (PC && range_bad) atomicOr(a.status, kStatusRange);
    }
    sync_for_mma();
    // ---- D1 = [K~; Q~] K^^T ;  [Z | O_a] = S' [K~; Q~]^T
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t ka = (kk >> 2) * LY::kKQBlk + (kk & 3) * 32;
        const uint32_t kh = (kk >> 2) * LY::kKHBlk + (kk & 3) * 32;
        const uint64_t ah = sdesc_sw128(s_kqh + ka, 16, 1024), al = sdesc_sw128(s_kql + ka, 16, 1024);
        mma_bf16_ss(tm + TC::D1, ah, sdesc_sw128(s_khh + kh, 16, 1024), ID_D1, kk > 0);
        mma_bf16_ss(tm + TC::D1, ah, sdesc_sw128(s_khl + kh, 16, 1024), ID_D1, 1);
        mma_bf16_ss(tm + TC::D1, al, sdesc_sw128(s_khh + kh, 16, 1024), ID_D1, 1);
        mma_ts(tm + TC::ZO, tm + TC::SH + 8 * kk, ah, ID_ZO, kk > 0);
        mma_ts(tm + TC::ZO, tm + TC::SH + 8 * kk, al, ID_ZO, 1);
        mma_ts(tm + TC::ZO, tm + TC::SL + 8 * kk, ah, ID_ZO, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    // ---- A (fp32, over K^) and P (hi / lo tiles) from D1; U's right-hand
    //      side V^T - zf Z into TMEM; S <- S Diag(e^{gl})
    if (lq < 2) {  // TMEM lanes 0-63: rows of A, columns 32 hs ..
      if (!add) {
      const int r = i;
      const float br = betav[r], gr = gcs[r];
      {
        const int hp = hs;
        float x[32];
        tmem_ld32(lb + TC::D1 + 32 * hp, x);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int s = 32 * hp + 4 * e4 + e;
            const float gam = PC ? 1.f : __expf(gr - gcs[s]);
            y[e] = (s < r && r < L) ? br * x[4 * e4 + e] * gam : 0.f;
          }
          Af4[r * 16 + ((8 * hp + e4) ^ (r & 15))] = make_float4(y[0], y[1], y[2], y[3]);
        }
      }
      }
    } else {  // TMEM lanes 64-127: rows of P, columns 32 hs ..
      const int r = i - 64;
      const float gr = gcs[r];
      {
        const int hp = hs;
        float x[32], hi[32], lo[32];
        tmem_ld32(lb + TC::D1 + 32 * hp, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int s = 32 * hp + e;
          const float gam = PC ? 1.f : __expf(gr - gcs[s]);
          split_bf16((s <= r && r < L) ? x[e] * gam : 0.f, hi[e], lo[e]);
        }
        st_row32(sm + LY::PP_HI, r, hp, hi);
        st_row32(sm + LY::PP_LO, r, hp, lo);
      }
    }
    {  // rows 32 hs .. 32 hs + 31 of this lane; all reads before any write
      float z[32];
      tmem_ld32(lb + TC::ZO + 32 * hs, z);
      const int ic = i < dv ? i : 0;
      float vr[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int r = 32 * hs + e;
        vr[e] = ld1<BF>(a.v, (tok0 + (size_t)(r < L ? r : 0) * H) * dv + ic);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int r = 32 * hs + e;
        z[e] = ((r < L && i < dv) ? vr[e] : 0.f) - (add ? 0.f : zf[r] * z[e]);
      }
      __syncthreads();
      tmem_put_split32(lb + TC::ZO + 16 * hs, lb + TC::ZO + 32 + 16 * hs, z);
    }
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TC::S + 32 * q, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= egl[32 * q + e];
      tmem_st32(lb + TC::S + 32 * q, x);
    }
    tmem_wait_st();
    __syncthreads();
    // ---- T = (I + A)^{-1} Diag(beta): column c by forward substitution
    //      (additive writes: T = I, U = V, none of this)
    if (!add) {
    if (t < 64) {  // Y over the per-channel decays (read only before D1)
      const int cl = t;
      float *Y = gcm;
      block_solve<1>(Af4, Y, cl);
      const float bc = betav[cl];
#pragma unroll 8
      for (int r = 0; r < C; ++r) {
        float hi, lo;
        split_bf16(Y[r * 64 + cl] * bc, hi, lo);
        const uint32_t off = sw128_off(r, cl);
        *reinterpret_cast<__nv_bfloat16 *>(sm + LY::TT_HI + off) = __float2bfloat16_rn(hi);
        *reinterpret_cast<__nv_bfloat16 *>(sm + LY::TT_LO + off) = __float2bfloat16_rn(lo);
      }
    }
    sync_for_mma();
    // ---- U^T = R T^T
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bh_ = sdesc_sw128(s_tth + kk * 32, 16, 1024);
        mma_ts(tm + TC::U, tm + TC::ZO + 8 * kk, bh_, ID_64, kk > 0);
        mma_ts(tm + TC::U, tm + TC::ZO + 8 * kk, sdesc_sw128(s_ttl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TC::U, tm + TC::ZO + 32 + 8 * kk, bh_, ID_64, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    {  // rows 32 hs .. of this lane; all reads before any write
      float u[32];
      tmem_ld32(lb + TC::U + 32 * hs, u);
      __syncthreads();
      tmem_put_split32(lb + TC::U + 16 * hs, lb + TC::U + 32 + 16 * hs, u);
    }
    }  // !add
    sync_for_mma();
    // ---- O_b = U^T P^T (over D1) ;  S += U^T (K e^{gl - gc})
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t ucol = add ? TC::ZO : TC::U;  // U^T (= V^T for additive writes)
        const uint32_t uh = tm + ucol + 8 * kk, ul = tm + ucol + 32 + 8 * kk;
        const uint64_t ph_ = sdesc_sw128(s_pph + kk * 32, 16, 1024);
        const uint64_t kb_ = sdesc_sw128(s_kbh + kk * 32, 16, 1024);
        mma_ts(tm + TC::D1, uh, ph_, ID_64, kk > 0);
        mma_ts(tm + TC::D1, uh, sdesc_sw128(s_ppl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TC::D1, ul, ph_, ID_64, 1);
        mma_ts(tm + TC::S, uh, kb_, ID_S, 1);
        mma_ts(tm + TC::S, uh, sdesc_sw128(s_kbl + kk * 32, 16, 1024), ID_S, 1);
        mma_ts(tm + TC::S, ul, kb_, ID_S, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    // ---- o_r = zf_r O_a + O_b (lane = value channel; rows 32 hs ..)
    {
      const int hp = hs;
      float oa[32], ob[32];
      tmem_ld32(lb + TC::ZO + 64 + 32 * hp, oa);
      tmem_ld32(lb + TC::D1 + 32 * hp, ob);
      if (i < dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r = 32 * hp + e;
          if (r < L) st1<BF>(a.o, (tok0 + (size_t)r * H) * dv + i, zf[r] * oa[e] + ob[e]);
        }
      }
    }
    __syncthreads();  // the vectors and tiles of this chunk are read
  }
  if (ok && a.S_T) {
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TC::S + 32 * q, x);
      if (i < dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = 32 * q + e;
          if (j < dk) a.S_T[((size_t)bh * dv + i) * dk + j] = x[e];
        }
      }
    }
  }
  if (!ok && t == 0) atomicOr(a.status, kStatusTimeout);
  if (t == 0) {  // every issued MMA has completed before TMEM is released
    mma_commit(bar);
    mbar_wait_bounded(bar, ph, kWaitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

template <int DK, bool PC, bool BF>
cudaError_t launch_split(const ChunkArgs &a, cudaStream_t stream) {
  auto kern = gdr_chunk_split_kernel<DK, PC, BF>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Layout<DK>::bytes);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(a.B * a.H), kThreadsD, Layout<DK>::bytes, stream>>>(a);
  return cudaGetLastError();
}


// ====================================================================== DPLR
// S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T,  o_t = S_t q_t
// ("Decoding Hybrid Linear Attention Architectures", section 3 item 5),
// chunked as that page's section 5 chunks the delta rule.  With e_r the
// decay from the chunk start (e_{-1} = 1), the low-rank reads x_r = S_{r-1}
// a_r of one chunk solve a unit lower-triangular system,
//   X^T = (S_0 A^^T + V^T Lk^T) T^T,  T = (I - Lb)^{-1},
//   Lb = strict_tril(A^ B^^T),  Lk = strict_tril(A^ K^^T),
//   a^_r = a_r e_{r-1},  b^_s = b_s / e_s,  k^_s = k_s / e_s,
// and then, with q~_r = q_r e_r,
//   O^T = S_0 Q~^T + X^T tril_incl(Q~ B^^T)^T + V^T tril_incl(Q~ K^^T)^T
//   S   = S_0 Diag(e_L) + X^T (B e_L / e) + V^T (K e_L / e).
// The four intra-chunk products come from one MMA group,
// [A^; Q~] [B^; K^]^T (M = 128, N = 128), and S_0 [A^; Q~]^T gives both
// state reads; the decay factors follow the delta-rule kernel above (per
// channel around the row-31 reference m, with the same range bound; a
// scalar gate's pairwise factors on the products).  Operands are split into
// two bf16 terms and products into three MMAs as above.
template <int DK>
struct DLayout {
  static constexpr uint32_t kBlk = 128 * 128;  // 128 rows x 64 bf16
  static constexpr uint32_t AQ_HI = 0, AQ_LO = AQ_HI + (DK / 64) * kBlk;
  static constexpr uint32_t BK_HI = AQ_LO + (DK / 64) * kBlk, BK_LO = BK_HI + (DK / 64) * kBlk;
  // after D1: Lb (fp32) and the Lk, P_b, P_k tiles over [A^; Q~] when it is
  // large enough (DK = 128), else in their own region; the transposed
  // B-bar, K-bar tiles over [B^; K^]
  static constexpr uint32_t POST = DK == 128 ? AQ_HI : BK_LO + (DK / 64) * kBlk;
  static constexpr uint32_t LB = POST, LK_HI = POST + 16384, LK_LO = LK_HI + 8192,
                            PB_HI = LK_LO + 8192, PB_LO = PB_HI + 8192, PK_HI = PB_LO + 8192,
                            PK_LO = PK_HI + 8192;
  static constexpr uint32_t BB_HI = BK_HI, BB_LO = BB_HI + DK * 128, KB_HI = BB_LO + DK * 128,
                            KB_LO = KB_HI + DK * 128;
  static constexpr uint32_t TT_HI = DK == 128 ? BK_LO + (DK / 64) * kBlk : PK_LO + 8192,
                            TT_LO = TT_HI + 8192;
  static constexpr uint32_t GC = TT_LO + 8192;
  static constexpr uint32_t VEC = GC + 64 * DK * 4;  // 768 floats
  static constexpr uint32_t BAR = VEC + 768 * 4, MISC = BAR + 16, END = MISC + 16;
  static constexpr size_t bytes = END + 1024;
  static_assert(PK_LO + 8192 <= (DK == 128 ? BK_HI : TT_HI), "post-D1 tiles fit");
  static_assert(KB_LO + DK * 128 <= BK_HI + 2 * (DK / 64) * kBlk, "B-bar, K-bar fit");
  static_assert(bytes <= 232448, "shared memory budget");
};

template <int DK, bool PC, bool BF>
__global__ void __launch_bounds__(kThreadsD, 1) gdr_dplr_split_kernel(DplrChunkArgs p) {
  using LY = DLayout<DK>;
  // TMEM: S [DK], S' hi / lo [DK/2 each], D1 [128] (then W / X in its first
  // 64 columns and V^T hi | lo in the last 64), ZO [128] (Z_a, then U's
  // right-hand side, then O_b, in the first 64; O_a in the last 64)
  constexpr uint32_t TS = 0, TSH = DK, TSL = DK + DK / 2, TD1 = 2 * DK, TZO = 2 * DK + 128;
  static_assert(TZO + 128 <= 512, "TMEM columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  // 8 warps: warp w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 (value
  // channels) and split that lane quarter's columns or rows between them (hs)
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, lq = warp & 3, hs = warp >> 2;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H, H = p.H;
  const int dk = p.dk, dv = p.dv;
  const int n = (p.T + C - 1) / C;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + LY::BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + LY::MISC);
  float *vec = reinterpret_cast<float *>(sm + LY::VEC);
  float *gcs = vec;         // [64] scalar gate: cumulative log decay
  float *zfo = vec + 64;    // [64] e^{gc_r} (scalar gate) or 1
  float *ebar = vec + 128;  // [64] scalar gate: e^{gl - gc_r}
  float *zfa = vec + 192;   // [64] e^{gc_{r-1}} (scalar gate) or 1
  float *mref = vec + 256, *em = vec + 384, *egl = vec + 512, *glv = vec + 640;  // [128] each
  float *gcm = reinterpret_cast<float *>(sm + LY::GC);  // [64][DK]
  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  const uint32_t lb = tm + ((uint32_t)(lq * 32) << 16);
  const int i = lq * 32 + lane;  // value channel (TMEM lane)

#pragma unroll 1
  for (int q = hs; q < DK / 32; q += 2) {
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = 32 * q + e;
      x[e] = (p.S0 && i < dv && j < dk) ? p.S0[((size_t)bh * dv + i) * dk + j] : 0.f;
    }
    tmem_st32(lb + TS + 32 * q, x);
  }
  tmem_wait_st();

  constexpr uint32_t ID_128 = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t ID_64 = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_S = idesc_bf16(128, DK, 0, 0);
  const uint32_t s_aqh = smem_u32(sm + LY::AQ_HI), s_aql = smem_u32(sm + LY::AQ_LO);
  const uint32_t s_bkh = smem_u32(sm + LY::BK_HI), s_bkl = smem_u32(sm + LY::BK_LO);
  const uint32_t s_lkh = smem_u32(sm + LY::LK_HI), s_lkl = smem_u32(sm + LY::LK_LO);
  const uint32_t s_pbh = smem_u32(sm + LY::PB_HI), s_pbl = smem_u32(sm + LY::PB_LO);
  const uint32_t s_pkh = smem_u32(sm + LY::PK_HI), s_pkl = smem_u32(sm + LY::PK_LO);
  const uint32_t s_bbh = smem_u32(sm + LY::BB_HI), s_bbl = smem_u32(sm + LY::BB_LO);
  const uint32_t s_kbh = smem_u32(sm + LY::KB_HI), s_kbl = smem_u32(sm + LY::KB_LO);
  const uint32_t s_tth = smem_u32(sm + LY::TT_HI), s_ttl = smem_u32(sm + LY::TT_LO);
  float4 *Lb4 = reinterpret_cast<float4 *>(sm + LY::LB);  // [64][16 float4], swizzled

  uint32_t ph = 0;
  bool ok = true;
  auto mma_wait = [&]() {
    if (t == 0) mma_commit(bar);
    ok = wait_all(bar, ph, ok);
    ph ^= 1;
    tc_fence_after();
  };

#pragma unroll 1
  for (int c = 0; c < n && ok; ++c) {
    const int t0 = c * C, L = min(C, p.T - t0);
    const size_t tok0 = ((size_t)b * p.T + t0) * H + h;
    // ---- gates
    if (PC) {
      if (t < DK) {
        const int j = t;
        float acc = 0.f, m = 0.f;
#pragma unroll 8
        for (int r = 0; r < C; ++r) {
          acc += (r < L && j < dk) ? p.g[(tok0 + (size_t)r * H) * dk + j] : 0.f;
          gcm[r * DK + j] = acc;
          if (r == 31) m = acc;
        }
        mref[j] = m;
        em[j] = __expf(m);
        egl[j] = __expf(acc);
        glv[j] = acc;
      }
      if (t < 64) {
        zfo[t] = 1.f;
        zfa[t] = 1.f;
      }
    } else if (warp == 0) {
      float x0 = lane < L ? p.g[tok0 + (size_t)lane * H] : 0.f;
      float x1 = lane + 32 < L ? p.g[tok0 + (size_t)(lane + 32) * H] : 0.f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
        if (lane >= off) {
          x0 += y0;
          x1 += y1;
        }
      }
      const float c31 = __shfl_sync(0xffffffffu, x0, 31);  // every lane takes part
      x1 += c31;
      const float gl = __shfl_sync(0xffffffffu, x1, 31);
      const float p0 = __shfl_up_sync(0xffffffffu, x0, 1), p1 = __shfl_up_sync(0xffffffffu, x1, 1);
      const float x0m = lane == 0 ? 0.f : p0;  // gc_{r-1}, r = lane
      const float x1m = lane == 0 ? c31 : p1;  // r = lane + 32
      gcs[lane] = x0;
      gcs[lane + 32] = x1;
      zfo[lane] = __expf(x0);
      zfo[lane + 32] = __expf(x1);
      zfa[lane] = __expf(x0m);
      zfa[lane + 32] = __expf(x1m);
      ebar[lane] = __expf(gl - x0);
      ebar[lane + 32] = __expf(gl - x1);
#pragma unroll
      for (int e = 0; e < 4; ++e) egl[lane + 32 * e] = __expf(gl);
    }
    __syncthreads();
    // ---- S' = S Diag(e^{m}) as hi / lo bf16 in TMEM
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TS + 32 * q, x);
      uint32_t hu[16], lu[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float f0 = PC ? em[32 * q + 2 * e] : 1.f, f1 = PC ? em[32 * q + 2 * e + 1] : 1.f;
        float h0, l0, h1, l1;
        split_bf16(x[2 * e] * f0, h0, l0);
        split_bf16(x[2 * e + 1] * f1, h1, l1);
        hu[e] = pack_bf16(h0, h1);
        lu[e] = pack_bf16(l0, l1);
      }
      tmem_st16u(lb + TSH + 16 * q, hu);
      tmem_st16u(lb + TSL + 16 * q, lu);
    }
    // ---- [A^; Q~] and [B^; K^] tiles: row r = t / 4, quarter t % 4 of the columns
    {
      const int r = t >> 2, hf = t & 3;
      bool range_bad = false;
#pragma unroll
      for (int g8 = 0; g8 < DK / 32; ++g8) {
        const int c0 = hf * (DK / 4) + 8 * g8;
        const bool valid = r < L && c0 < dk;
        const size_t off = in_off(tok0, r, c0, H, dk, valid);
        float ax[8], qx[8], bx[8], kx[8];
        ld8<BF>(p.a, off, ax);
        ld8<BF>(p.q, off, qx);
        ld8<BF>(p.b, off, bx);
        ld8<BF>(p.k, off, kx);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ax[e] = valid ? ax[e] : 0.f;
          qx[e] = valid ? qx[e] : 0.f;
          bx[e] = valid ? bx[e] : 0.f;
          kx[e] = valid ? kx[e] : 0.f;
        }
        if (PC) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = c0 + e;
            const float m = mref[j], gr = gcm[r * DK + j];
            const float xa = (r > 0 ? gcm[(r - 1) * DK + j] : 0.f) - m, xq = gr - m;
            const bool ia = fabsf(xa) <= kMaxExp, iq = fabsf(xq) <= kMaxExp;
            range_bad |= (!ia && ax[e] != 0.f) || (!iq && (qx[e] != 0.f || bx[e] != 0.f ||
                                                            kx[e] != 0.f));
            const float fa = ia ? __expf(xa) : 0.f, fq = iq ? __expf(xq) : 0.f,
                        fb = iq ? __expf(-xq) : 0.f;
            ax[e] *= fa;
            qx[e] *= fq;
            bx[e] *= fb;
            kx[e] *= fb;
          }
        }
        const uint32_t blk = (uint32_t)(c0 >> 6) * LY::kBlk, cc = (uint32_t)(c0 & 63);
        put8(sm + LY::AQ_HI + blk, sm + LY::AQ_LO + blk, sw128_off(r, cc), ax);
        put8(sm + LY::AQ_HI + blk, sm + LY::AQ_LO + blk, sw128_off(64 + r, cc), qx);
        put8(sm + LY::BK_HI + blk, sm + LY::BK_LO + blk, sw128_off(r, cc), bx);
        put8(sm + LY::BK_HI + blk, sm + LY::BK_LO + blk, sw128_off(64 + r, cc), kx);
      }
      if (PC && range_bad) atomicOr(p.status, kStatusRange);
    }
    sync_for_mma();
    // ---- D1 = [A^; Q~] [B^; K^]^T ;  [Z_a | O_a] = S' [A^; Q~]^T
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * LY::kBlk + (kk & 3) * 32;
        const uint64_t ah = sdesc_sw128(s_aqh + ko, 16, 1024), al = sdesc_sw128(s_aql + ko, 16, 1024);
        const uint64_t bh_ = sdesc_sw128(s_bkh + ko, 16, 1024);
        mma_bf16_ss(tm + TD1, ah, bh_, ID_128, kk > 0);
        mma_bf16_ss(tm + TD1, ah, sdesc_sw128(s_bkl + ko, 16, 1024), ID_128, 1);
        mma_bf16_ss(tm + TD1, al, bh_, ID_128, 1);
        mma_ts(tm + TZO, tm + TSH + 8 * kk, ah, ID_128, kk > 0);
        mma_ts(tm + TZO, tm + TSH + 8 * kk, al, ID_128, 1);
        mma_ts(tm + TZO, tm + TSL + 8 * kk, ah, ID_128, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    // ---- from D1: Lb (fp32), Lk, P_b, P_k (hi / lo tiles)
    if (lq < 2) {  // rows 0-63: Lb (hs = 0) and Lk (hs = 1)
      const int r = i;
      const float gr = r > 0 ? gcs[r - 1] : 0.f;
#pragma unroll 1
      for (int hp = 2 * hs; hp < 2 * hs + 2; ++hp) {  // D1 columns 32 hp .. 32 hp + 31
        float x[32];
        tmem_ld32(lb + TD1 + 32 * hp, x);
        float hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int s = 32 * (hp & 1) + e;
          const float gam = PC ? 1.f : __expf(gr - gcs[s]);
          x[e] = (s < r && r < L) ? x[e] * gam : 0.f;
          split_bf16(x[e], hi[e], lo[e]);
        }
        if (hp < 2) {
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4)
            Lb4[r * 16 + ((8 * hp + e4) ^ (r & 15))] =
                make_float4(x[4 * e4], x[4 * e4 + 1], x[4 * e4 + 2], x[4 * e4 + 3]);
        } else {
          st_row32(sm + LY::LK_HI, r, hp & 1, hi);
          st_row32(sm + LY::LK_LO, r, hp & 1, lo);
        }
      }
    } else {  // rows 64-127: P_b (hs = 0) and P_k (hs = 1)
      const int r = i - 64;
      const float gr = gcs[r];
#pragma unroll 1
      for (int hp = 2 * hs; hp < 2 * hs + 2; ++hp) {
        float x[32], hi[32], lo[32];
        tmem_ld32(lb + TD1 + 32 * hp, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int s = 32 * (hp & 1) + e;
          const float gam = PC ? 1.f : __expf(gr - gcs[s]);
          split_bf16((s <= r && r < L) ? x[e] * gam : 0.f, hi[e], lo[e]);
        }
        st_row32(sm + (hp < 2 ? LY::PB_HI : LY::PK_HI), r, hp & 1, hi);
        st_row32(sm + (hp < 2 ? LY::PB_LO : LY::PK_LO), r, hp & 1, lo);
      }
    }
    __syncthreads();  // every lane's D1 columns 64-127 read before V^T goes there
    {  // V^T (lane = value channel) as hi | lo into D1 columns 64-127; rows 32 hs ..
      float vt[32];
      const int ic = i < dv ? i : 0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int r = 32 * hs + e;
        vt[e] = ld1<BF>(p.v, (tok0 + (size_t)(r < L ? r : 0) * H) * dv + ic);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) vt[e] = (32 * hs + e < L && i < dv) ? vt[e] : 0.f;
      tmem_put_split32(lb + TD1 + 64 + 16 * hs, lb + TD1 + 96 + 16 * hs, vt);
    }
    {  // (B e^{gl - gc})^T and (K e^{gl - gc})^T over [B^; K^] (dead after D1)
      const int r = t >> 2, hf = t & 3;
#pragma unroll
      for (int g8 = 0; g8 < DK / 32; ++g8) {
        const int c0 = hf * (DK / 4) + 8 * g8;
        const bool valid = r < L && c0 < dk;
        const size_t off = in_off(tok0, r, c0, H, dk, valid);
        float bx[8], kx[8];
        ld8<BF>(p.b, off, bx);
        ld8<BF>(p.k, off, kx);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          bx[e] = valid ? bx[e] : 0.f;
          kx[e] = valid ? kx[e] : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = c0 + e;
          const float f = PC ? __expf(glv[j] - gcm[r * DK + j]) : ebar[r];
          float hi, lo;
          const uint32_t off = sw128_off(j, r);
          split_bf16(bx[e] * f, hi, lo);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::BB_HI + off) = __float2bfloat16_rn(hi);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::BB_LO + off) = __float2bfloat16_rn(lo);
          split_bf16(kx[e] * f, hi, lo);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::KB_HI + off) = __float2bfloat16_rn(hi);
          *reinterpret_cast<__nv_bfloat16 *>(sm + LY::KB_LO + off) = __float2bfloat16_rn(lo);
        }
      }
    }
    sync_for_mma();
    // ---- W = V^T Lk^T (over D1 columns 0-63)
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t lh = sdesc_sw128(s_lkh + kk * 32, 16, 1024);
        mma_ts(tm + TD1, tm + TD1 + 64 + 8 * kk, lh, ID_64, kk > 0);
        mma_ts(tm + TD1, tm + TD1 + 64 + 8 * kk, sdesc_sw128(s_lkl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TD1, tm + TD1 + 96 + 8 * kk, lh, ID_64, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    // ---- R = zfa Z_a + W -> hi | lo over Z_a;  S <- S Diag(e^{gl})
    {  // rows 32 hs .. 32 hs + 31 of this lane; all reads before any write
      float z[32], w[32];
      tmem_ld32(lb + TZO + 32 * hs, z);
      tmem_ld32(lb + TD1 + 32 * hs, w);
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = zfa[32 * hs + e] * z[e] + w[e];
      __syncthreads();
      tmem_put_split32(lb + TZO + 16 * hs, lb + TZO + 32 + 16 * hs, z);
    }
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TS + 32 * q, x);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= egl[32 * q + e];
      tmem_st32(lb + TS + 32 * q, x);
    }
    tmem_wait_st();
    // ---- T = (I - Lb)^{-1}: column c by forward substitution
    if (t < 64) {  // Y over the per-channel decays (read only before this)
      const int cl = t;
      float *Y = gcm;
      block_solve<-1>(Lb4, Y, cl);
#pragma unroll 8
      for (int r = 0; r < C; ++r) {
        float hi, lo;
        split_bf16(Y[r * 64 + cl], hi, lo);
        const uint32_t off = sw128_off(r, cl);
        *reinterpret_cast<__nv_bfloat16 *>(sm + LY::TT_HI + off) = __float2bfloat16_rn(hi);
        *reinterpret_cast<__nv_bfloat16 *>(sm + LY::TT_LO + off) = __float2bfloat16_rn(lo);
      }
    }
    sync_for_mma();
    // ---- X^T = R T^T (over D1 columns 0-63)
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t th = sdesc_sw128(s_tth + kk * 32, 16, 1024);
        mma_ts(tm + TD1, tm + TZO + 8 * kk, th, ID_64, kk > 0);
        mma_ts(tm + TD1, tm + TZO + 8 * kk, sdesc_sw128(s_ttl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TD1, tm + TZO + 32 + 8 * kk, th, ID_64, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    {  // rows 32 hs .. 32 hs + 31 of this lane; all reads before any write
      float x[32];
      tmem_ld32(lb + TD1 + 32 * hs, x);
      __syncthreads();
      tmem_put_split32(lb + TD1 + 16 * hs, lb + TD1 + 32 + 16 * hs, x);
    }
    sync_for_mma();
    // ---- O_b = X^T P_b^T + V^T P_k^T (over ZO columns 0-63);
    //      S += X^T (B e^{gl - gc}) + V^T (K e^{gl - gc})
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t xh = tm + TD1 + 8 * kk, xl = tm + TD1 + 32 + 8 * kk;
        const uint32_t vh = tm + TD1 + 64 + 8 * kk, vl = tm + TD1 + 96 + 8 * kk;
        const uint64_t pb = sdesc_sw128(s_pbh + kk * 32, 16, 1024);
        const uint64_t pk = sdesc_sw128(s_pkh + kk * 32, 16, 1024);
        const uint64_t bb = sdesc_sw128(s_bbh + kk * 32, 16, 1024);
        const uint64_t kb = sdesc_sw128(s_kbh + kk * 32, 16, 1024);
        mma_ts(tm + TZO, xh, pb, ID_64, kk > 0);
        mma_ts(tm + TZO, xh, sdesc_sw128(s_pbl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TZO, xl, pb, ID_64, 1);
        mma_ts(tm + TZO, vh, pk, ID_64, 1);
        mma_ts(tm + TZO, vh, sdesc_sw128(s_pkl + kk * 32, 16, 1024), ID_64, 1);
        mma_ts(tm + TZO, vl, pk, ID_64, 1);
        mma_ts(tm + TS, xh, bb, ID_S, 1);
        mma_ts(tm + TS, xh, sdesc_sw128(s_bbl + kk * 32, 16, 1024), ID_S, 1);
        mma_ts(tm + TS, xl, bb, ID_S, 1);
        mma_ts(tm + TS, vh, kb, ID_S, 1);
        mma_ts(tm + TS, vh, sdesc_sw128(s_kbl + kk * 32, 16, 1024), ID_S, 1);
        mma_ts(tm + TS, vl, kb, ID_S, 1);
      }
    }
    mma_wait();
    if (!ok) break;
    // ---- o_r = zfo_r O_a + O_b (rows 32 hs .. 32 hs + 31)
    {
      const int hp = hs;
      float oa[32], ob[32];
      tmem_ld32(lb + TZO + 64 + 32 * hp, oa);
      tmem_ld32(lb + TZO + 32 * hp, ob);
      if (i < dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r = 32 * hp + e;
          if (r < L) st1<BF>(p.o, (tok0 + (size_t)r * H) * dv + i, zfo[r] * oa[e] + ob[e]);
        }
      }
    }
    __syncthreads();
  }
  if (ok && p.S_T) {
#pragma unroll 1
    for (int q = hs; q < DK / 32; q += 2) {
      float x[32];
      tmem_ld32(lb + TS + 32 * q, x);
      if (i < dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = 32 * q + e;
          if (j < dk) p.S_T[((size_t)bh * dv + i) * dk + j] = x[e];
        }
      }
    }
  }
  if (!ok && t == 0) atomicOr(p.status, kStatusTimeout);
  if (t == 0) {
    mma_commit(bar);
    mbar_wait_bounded(bar, ph, kWaitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

template <int DK, bool PC, bool BF>
cudaError_t launch_dplr_split(const DplrChunkArgs &a, cudaStream_t stream) {
  auto kern = gdr_dplr_split_kernel<DK, PC, BF>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)DLayout<DK>::bytes);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(a.B * a.H), kThreadsD, DLayout<DK>::bytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool chunk_split_supports(const ChunkArgs &a) {
  const bool dims = (a.dk == 32 || a.dk == 64 || a.dk == 128) &&
                    (a.dv == 32 || a.dv == 64 || a.dv == 128);
  return dims && !a.stash_x && !a.stash_v && !a.stash_t && a.s0_seg == 0 && !a.s0_identity &&
         a.seg_n == 0 &&
         !a.zero_v && a.write_o && a.skip_stage_chunk < 0 && (!a.prologue || a.gate_scale);
}

cudaError_t launch_chunk_split(const ChunkArgs &a, cudaStream_t stream) {
  if (!chunk_split_supports(a)) return cudaErrorNotSupported;
  if (a.B * a.H == 0) return cudaSuccess;
  const int key = (a.dk == 128 ? 4 : 0) | (a.per_channel ? 2 : 0) | (a.bf16 ? 1 : 0);
  switch (key) {
    case 0: return launch_split<64, false, false>(a, stream);
    case 1: return launch_split<64, false, true>(a, stream);
    case 2: return launch_split<64, true, false>(a, stream);
    case 3: return launch_split<64, true, true>(a, stream);
    case 4: return launch_split<128, false, false>(a, stream);
    case 5: return launch_split<128, false, true>(a, stream);
    case 6: return launch_split<128, true, false>(a, stream);
    default: return launch_split<128, true, true>(a, stream);
  }
}

cudaError_t launch_dplr_chunk(const DplrChunkArgs &a, cudaStream_t stream) {
  const bool dims = (a.dk == 32 || a.dk == 64 || a.dk == 128) &&
                    (a.dv == 32 || a.dv == 64 || a.dv == 128);
  if (!dims) return cudaErrorNotSupported;
  if (a.B * a.H == 0) return cudaSuccess;
  const int key = (a.dk == 128 ? 4 : 0) | (a.per_channel ? 2 : 0) | (a.bf16 ? 1 : 0);
  switch (key) {
    case 0: return launch_dplr_split<64, false, false>(a, stream);
    case 1: return launch_dplr_split<64, false, true>(a, stream);
    case 2: return launch_dplr_split<64, true, false>(a, stream);
    case 3: return launch_dplr_split<64, true, true>(a, stream);
    case 4: return launch_dplr_split<128, false, false>(a, stream);
    case 5: return launch_dplr_split<128, false, true>(a, stream);
    case 6: return launch_dplr_split<128, true, false>(a, stream);
    default: return launch_dplr_split<128, true, true>(a, stream);
  }
}

}  // namespace gdr
