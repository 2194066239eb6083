// Chunkwise gated delta-rule forward on the sm_100a tensor cores (tcgen05),
// bf16 q/k/v, fp32 gates and state, d_k = d_v = 128, scalar gate, C = 64.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5
// (inter-chunk state recursion S <- decay S + (decay K)^T (U - W S),
// intra-chunk output (decay Q) S + tril(...)(U - W S), log-space gates) and
// the WY/UT representation of the delta rule ("Linear Attention Variants",
// DeltaNet section).  Written in the state's own orientation (S is d_v x d_k,
// one TMEM lane per value channel i), for one chunk of C = 64 tokens with
// gc_r = cumulative log decay from the chunk start:
//
//   D1   = [K; Q] K^T                      (tcgen05, M=128 N=64 K=128)
//   A    = strict_tril(beta_r D1_KK[r][s] e^{gc_r - gc_s})
//   P    = tril_incl(D1_QK[r][s] e^{gc_r - gc_s})       -> bf16, smem
//   Y    = (I + A)^{-1}   (blocked forward substitution, fp32 CUDA cores)
//   T    = Y Diag(beta),  T' = T Diag(e^{gc})            -> bf16, smem
//   U^T  = V^T T^T,  W^T = K^T T'^T        (tcgen05, M=128 N=64 K=64)
//   V'^T = U^T - S_b W^T                   (tcgen05, negated A, K=128)
//   O^T  = Diag(e^{gc}) (S_b Q^T) + V'^T P^T
//   S    = e^{gc_last} S + (V'^T Diag(e^{gc_last - gc})) K   (fp32 TMEM acc)
//
// S_b is the bf16 copy of the fp32 state used as an MMA operand.  Every
// exponent formed is <= 0, so no gate can overflow this path.
//
// Structure: one CTA per (b, h); warps 0-3 own TMEM lanes 0-127 and do all
// epilogue / CUDA-core work (thread 0 issues the MMAs); warp 4 is the
// producer: TMA (no multicast) for the K, Q, V tiles of the next chunks
// (two stages) and plain loads for g and beta.  Every wait is bounded: on
// time-out the kernel sets the device status word and unwinds.
#include <cudaTypedefs.h>

#include <mutex>

#include "gdr_internal.cuh"
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kCompute = 128;
constexpr int kThreads = kCompute + 32;
constexpr int kStages = 2;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kTileBytes = 64 * 128;    // one 64 x 64 bf16 tile
constexpr uint32_t kStageTx = 6 * kTileBytes;

// Shared-memory layout (byte offsets from a 1024-byte aligned base).
struct Lay {
  static constexpr uint32_t KQ = 0;                       // per stage [K_h0|Q_h0|K_h1|Q_h1]
  static constexpr uint32_t V = KQ + kStages * 4 * kTileBytes;  // per stage [V_h0|V_h1]
  static constexpr uint32_t T = V + kStages * 2 * kTileBytes;   // T   K-major [r][s]
  static constexpr uint32_t TP = T + kTileBytes;                // T'  K-major [r][s]
  static constexpr uint32_t P = TP + kTileBytes;                // P   K-major [r][s]
  static constexpr uint32_t WT = P + kTileBytes;                // W^T MN-major [dk][C]
  static constexpr uint32_t SB = WT + 2 * kTileBytes;           // S_b K-major [dv][dk], 2 halves
  static constexpr uint32_t VP = SB + 4 * kTileBytes;           // V'^T K-major [dv][C]
  static constexpr uint32_t VPD = VP + 2 * kTileBytes;          // decayed V'^T
  static constexpr uint32_t AF = VPD + 2 * kTileBytes;          // fp32 A/Y [64][65]; O staging
  static constexpr uint32_t R = AF + 64 * 65 * 4;               // fp32 [16][49] inverse scratch
  static constexpr uint32_t GS = R + 3200;                      // per stage g[64], beta[64]
  static constexpr uint32_t VEC = GS + kStages * 512;           // gc[64], eg[64], egl[64]
  static constexpr uint32_t BAR = VEC + 768;                    // full[2], empty[2], mma
  static constexpr uint32_t MISC = BAR + 64;                    // tmem base, abort flag
  static constexpr uint32_t END = MISC + 16;
};
static_assert(Lay::AF % 1024 == 0, "tile alignment");
constexpr size_t kSmemBytes = Lay::END + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM column map (512 columns allocated; 1 CTA per SM).
constexpr uint32_t TM_S = 0, TM_D1 = 128, TM_UV = 192, TM_WT = 256, TM_OA = 320, TM_OB = 384;

constexpr uint32_t ID_D1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_U = idesc_bf16(128, 64, 1, 0);
constexpr uint32_t ID_VP = idesc_bf16(128, 64, 0, 1, /*neg_a=*/1);
constexpr uint32_t ID_O = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 1);

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&t);
}

// Write 64 fp32 values as one bf16 row (128 bytes) of a 128B-swizzled tile.
__device__ __forceinline__ void st_row64_sw128(uint8_t *tile, int row, const float *x) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    uint4 u;
    u.x = pack_bf16(x[8 * ch + 0], x[8 * ch + 1]);
    u.y = pack_bf16(x[8 * ch + 2], x[8 * ch + 3]);
    u.z = pack_bf16(x[8 * ch + 4], x[8 * ch + 5]);
    u.w = pack_bf16(x[8 * ch + 6], x[8 * ch + 7]);
    *reinterpret_cast<uint4 *>(tile + sw128_off(row, 8 * ch)) = u;
  }
}

// 64 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  float t[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    tmem_ld16(taddr + 16 * q, t);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[16 * q + i] = t[i];
  }
  tmem_wait_ld();
}

// All 128 compute threads: barrier that also ORs a predicate.
__device__ __forceinline__ bool bar_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void cbar() { named_bar_sync(1, kCompute); }

#ifdef GDR_TC_DEBUG
// Debug build only: stage values of one chunk of CTA 0 are copied out.
__device__ float *g_dbg = nullptr;
__device__ int g_dbg_chunk = 0;
#define DBG_ROW(off, ncol, src)                                               \
  do {                                                                        \
    if (g_dbg && blockIdx.x == 0 && c == g_dbg_chunk)                        \
      for (int _e = 0; _e < (ncol); ++_e) g_dbg[(off) + i * (ncol) + _e] = (src)[_e]; \
  } while (0)
#else
#define DBG_ROW(off, ncol, src) \
  do {                          \
  } while (0)
#endif

// (I + A)^{-1} in place for a strictly lower 64x64 fp32 matrix (row stride
// 65), by 16x16 blocks: diagonal blocks by forward substitution (warp w owns
// block w), then block rows b = 1..3:  Y_b = -D_bb sum_{k<b} A_bk Y_k.
__device__ void invert_unit_lower(float *AF, float *R, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  {
    const int w = warp, c = lane & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
    const float *Ab = AF + (16 * w) * 65 + 16 * w;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < i; ++k) acc += Ab[i * 65 + k] * x[k];
      if (i > c) x[i] = -acc;
    }
    __syncwarp();
    if (lane < 16) {
      float *Yb = AF + (16 * w) * 65 + 16 * w;
#pragma unroll
      for (int i = 0; i < 16; ++i) Yb[i * 65 + c] = x[i];
    }
  }
  cbar();
  for (int b = 1; b < 4; ++b) {
    const int ncol = 16 * b;
    for (int idx = tid; idx < 16 * ncol; idx += kCompute) {
      const int i = idx / ncol, c = idx % ncol, jb = c >> 4;
      const float *Arow = AF + (16 * b + i) * 65;
      float acc = 0.f;
      for (int m = 16 * jb; m < 16 * b; ++m) acc += Arow[m] * AF[m * 65 + c];
      R[i * 49 + c] = acc;
    }
    cbar();
    for (int idx = tid; idx < 16 * ncol; idx += kCompute) {
      const int i = idx / ncol, c = idx % ncol;
      const float *Drow = AF + (16 * b + i) * 65 + 16 * b;
      float acc = 0.f;
      for (int l = 0; l <= i; ++l) acc += Drow[l] * R[l * 49 + c];
      AF[(16 * b + i) * 65 + c] = -acc;
    }
    cbar();
  }
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// D += A(16x8, row) * B(8x8, col), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Same result as invert_unit_lower, with the off-diagonal block products on
// the warp-level tensor cores (TF32 operands rounded to nearest, fp32
// accumulation): for block row b, warp w computes 8-column tiles nt = w,
// w + 4, ... of R_b = sum_{k<b} A_bk Y_k, then Y_b = -D_bb R_b.
__device__ void invert_unit_lower_mma(float *AF, float *R, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  {
    const int w = warp, c = lane & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
    const float *Ab = AF + (16 * w) * 65 + 16 * w;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < i; ++k) acc += Ab[i * 65 + k] * x[k];
      if (i > c) x[i] = -acc;
    }
    __syncwarp();
    if (lane < 16) {
      float *Yb = AF + (16 * w) * 65 + 16 * w;
#pragma unroll
      for (int i = 0; i < 16; ++i) Yb[i * 65 + c] = x[i];
    }
  }
  cbar();
  const int g = lane >> 2, t = lane & 3;
  for (int b = 1; b < 4; ++b) {
    const int ntiles = 2 * b;
    // phase 1: R_b tiles -> R [16][49]
    for (int nt = warp; nt < ntiles; nt += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = nt >> 1; k < b; ++k) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const int col = 16 * k + 8 * ks;
          uint32_t af[4], bf[2];
          af[0] = to_tf32(AF[(16 * b + g) * 65 + col + t]);
          af[1] = to_tf32(AF[(16 * b + g + 8) * 65 + col + t]);
          af[2] = to_tf32(AF[(16 * b + g) * 65 + col + t + 4]);
          af[3] = to_tf32(AF[(16 * b + g + 8) * 65 + col + t + 4]);
          bf[0] = to_tf32(AF[(col + t) * 65 + 8 * nt + g]);
          bf[1] = to_tf32(AF[(col + t + 4) * 65 + 8 * nt + g]);
          mma_tf32_16x8x8(acc, af, bf);
        }
      }
      R[g * 49 + 8 * nt + 2 * t] = acc[0];
      R[g * 49 + 8 * nt + 2 * t + 1] = acc[1];
      R[(g + 8) * 49 + 8 * nt + 2 * t] = acc[2];
      R[(g + 8) * 49 + 8 * nt + 2 * t + 1] = acc[3];
    }
    cbar();
    // phase 2: Y_b tile = -D_bb R_b tile  (D_bb sits in AF's diagonal block)
    for (int nt = warp; nt < ntiles; nt += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const int col = 16 * b + 8 * ks;
        uint32_t af[4], bf[2];
        af[0] = to_tf32(AF[(16 * b + g) * 65 + col + t]);
        af[1] = to_tf32(AF[(16 * b + g + 8) * 65 + col + t]);
        af[2] = to_tf32(AF[(16 * b + g) * 65 + col + t + 4]);
        af[3] = to_tf32(AF[(16 * b + g + 8) * 65 + col + t + 4]);
        bf[0] = to_tf32(R[(8 * ks + t) * 49 + 8 * nt + g]);
        bf[1] = to_tf32(R[(8 * ks + t + 4) * 49 + 8 * nt + g]);
        mma_tf32_16x8x8(acc, af, bf);
      }
      AF[(16 * b + g) * 65 + 8 * nt + 2 * t] = -acc[0];
      AF[(16 * b + g) * 65 + 8 * nt + 2 * t + 1] = -acc[1];
      AF[(16 * b + g + 8) * 65 + 8 * nt + 2 * t] = -acc[2];
      AF[(16 * b + g + 8) * 65 + 8 * nt + 2 * t + 1] = -acc[3];
    }
    cbar();
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gdr_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmO, ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int T = a.T, H = a.H;
  const int nchunks = (T + C - 1) / C;

  uint64_t *full = reinterpret_cast<uint64_t *>(sm + Lay::BAR);
  uint64_t *empty = full + 2;
  uint64_t *mmab = full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::MISC);
  volatile int *consumed = reinterpret_cast<volatile int *>(sm + Lay::MISC + 4);
  float *gcv = reinterpret_cast<float *>(sm + Lay::VEC);
  float *egv = gcv + 64;
  float *eglv = gcv + 128;
  float *AF = reinterpret_cast<float *>(sm + Lay::AF);
  float *Rs = reinterpret_cast<float *>(sm + Lay::R);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(mmab, 1);
    *consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int issued = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1;
      if (c >= kStages) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ((c >> 1) - 1) & 1, kWaitNs);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) atomicOr(a.status, kStatusTimeout);
          break;
        }
      }
      const int t0 = c * C;
      float *gs = reinterpret_cast<float *>(sm + Lay::GS + s * 512);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int r = lane + 32 * q, t = t0 + r;
        const size_t tok = ((size_t)b * T + t) * H + h;
        gs[r] = t < T ? a.g[tok] : 0.f;
        gs[64 + r] = t < T ? a.beta[tok] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kStageTx);
        uint8_t *kq = sm + Lay::KQ + s * 4 * kTileBytes;
        uint8_t *vv = sm + Lay::V + s * 2 * kTileBytes;
        tma_load_4d(kq + 0 * kTileBytes, &tmK, &full[s], 0, h, t0, b);
        tma_load_4d(kq + 1 * kTileBytes, &tmQ, &full[s], 0, h, t0, b);
        tma_load_4d(kq + 2 * kTileBytes, &tmK, &full[s], 64, h, t0, b);
        tma_load_4d(kq + 3 * kTileBytes, &tmQ, &full[s], 64, h, t0, b);
        tma_load_4d(vv + 0 * kTileBytes, &tmV, &full[s], 0, h, t0, b);
        tma_load_4d(vv + 1 * kTileBytes, &tmV, &full[s], 64, h, t0, b);
      }
      ++issued;
    }
    // Drain loads that were issued but never consumed (only after an abort).
    if (lane == 0) {
      for (int c = *consumed; c < issued; ++c) {
        if (!mbar_wait_bounded(&full[c & 1], (c >> 1) & 1, kWaitNs))
          atomicOr(a.status, kStatusTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    const int i = tid;  // TMEM lane = value channel (state row)
    const uint32_t lane_base = tm + ((uint32_t)(warp * 32) << 16);
    uint32_t mma_phase = 0;
    bool aborted = false;

    // Initial state: S0 row i -> TMEM (fp32) and S_b (bf16).
    {
      float x[64];
      for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          x[j] = a.S0 ? a.S0[((size_t)bh * DV + i) * DK + 64 * hh + j] : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float t[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] = x[16 * q + e];
          tmem_st16(lane_base + TM_S + 64 * hh + 16 * q, t);
        }
        st_row64_sw128(sm + Lay::SB + hh * 2 * kTileBytes, i, x);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
    }

    const uint32_t a_kq = smem_u32(sm + Lay::KQ);
    const uint32_t a_v = smem_u32(sm + Lay::V);
    const uint32_t a_t = smem_u32(sm + Lay::T), a_tp = smem_u32(sm + Lay::TP);
    const uint32_t a_p = smem_u32(sm + Lay::P), a_wt = smem_u32(sm + Lay::WT);
    const uint32_t a_sb = smem_u32(sm + Lay::SB), a_vp = smem_u32(sm + Lay::VP);
    const uint32_t a_vpd = smem_u32(sm + Lay::VPD);

    auto wait_mma = [&]() -> bool {
      bool ok = mbar_wait_bounded(mmab, mma_phase, kWaitNs);
      mma_phase ^= 1;
      const bool bad = bar_any(!ok);
      tc_fence_after();
      return !bad;
    };

    for (int c = 0; c < nchunks && !aborted; ++c) {
      const int s = c & 1, t0 = c * C;
      {
        const bool ok = mbar_wait_bounded(&full[s], (c >> 1) & 1, kWaitNs);
        if (bar_any(!ok)) { aborted = true; break; }
      }
      const float *gs = reinterpret_cast<const float *>(sm + Lay::GS + s * 512);
      const float *bs = gs + 64;
      const uint32_t kq = a_kq + s * 4 * kTileBytes;
      const uint32_t vv = a_v + s * 2 * kTileBytes;

      // cumulative log decay (warp 0), decay factors
      if (warp == 0) {
        float x0 = gs[lane], x1 = gs[lane + 32];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, off);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, off);
          if (lane >= off) { x0 += y0; x1 += y1; }
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const float gl = __shfl_sync(0xffffffffu, x1, 31);
        gcv[lane] = x0;
        gcv[lane + 32] = x1;
        egv[lane] = __expf(x0);
        egv[lane + 32] = __expf(x1);
        eglv[lane] = __expf(gl - x0);
        eglv[lane + 32] = __expf(gl - x1);
      }
      if (tid == 0) tma_store_wait_read0();  // O staging (aliases AF) is free again
      cbar();

      // ---- D1 = [K; Q] K^T
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          mma_bf16_ss(tm + TM_D1, sdesc_sw128(kq + off, 16, 1024),
                      sdesc_sw128(kq + off, 16, 1024), ID_D1, kk > 0);
        }
        mma_commit(mmab);
      }
      if (!wait_mma()) { aborted = true; break; }

      // ---- A (lanes 0-63) and P (lanes 64-127)
      {
        float x[64];
        tmem_ld64(lane_base + TM_D1, x);
        DBG_ROW(0, 64, x);
        const int r = i & 63;
        const float gr = gcv[r];
        if (i < 64) {
          const float br = bs[r];
#pragma unroll
          for (int s2 = 0; s2 < 64; ++s2)
            AF[r * 65 + s2] = (s2 < r) ? br * x[s2] * __expf(gr - gcv[s2]) : 0.f;
        } else {
#pragma unroll
          for (int s2 = 0; s2 < 64; ++s2) x[s2] = (s2 <= r) ? x[s2] * __expf(gr - gcv[s2]) : 0.f;
          st_row64_sw128(sm + Lay::P, r, x);
        }
      }
      cbar();
#ifdef GDR_TC_DEBUG
      if (i < 64) DBG_ROW(8192, 64, AF + i * 65);
      cbar();
#endif
      invert_unit_lower(AF, Rs, tid);
#ifdef GDR_TC_DEBUG
      if (i < 64) DBG_ROW(12288, 64, AF + i * 65);
#endif
      // ---- T = Y Diag(beta) and T' = T Diag(e^{gc}) as bf16 operands
      {
        const int r = i & 63;
        float x[64];
        if (i < 64) {
#pragma unroll
          for (int s2 = 0; s2 < 64; ++s2) x[s2] = AF[r * 65 + s2] * bs[s2];
          st_row64_sw128(sm + Lay::T, r, x);
        } else {
#pragma unroll
          for (int s2 = 0; s2 < 64; ++s2) x[s2] = AF[r * 65 + s2] * bs[s2] * egv[s2];
          st_row64_sw128(sm + Lay::TP, r, x);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      cbar();

      // ---- U^T = V^T T^T, W^T = K^T T'^T, O_a = S_b Q^T
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16_ss(tm + TM_UV, sdesc_sw128(vv + kk * 2048, kTileBytes, 1024),
                      sdesc_sw128(a_t + kk * 32, 16, 1024), ID_U, kk > 0);
          mma_bf16_ss(tm + TM_WT, sdesc_sw128(kq + kk * 2048, 2 * kTileBytes, 1024),
                      sdesc_sw128(a_tp + kk * 32, 16, 1024), ID_U, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          const uint32_t boff = kTileBytes + (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          mma_bf16_ss(tm + TM_OA, sdesc_sw128(a_sb + aoff, 16, 1024),
                      sdesc_sw128(kq + boff, 16, 1024), ID_O, kk > 0);
        }
        mma_commit(mmab);
      }
      if (!wait_mma()) { aborted = true; break; }

      // ---- W^T -> bf16 MN-major operand (row j = this thread's lane)
      {
        float x[64];
        tmem_ld64(lane_base + TM_WT, x);
        DBG_ROW(16384, 64, x);
#ifdef GDR_TC_DEBUG
        {
          float u[64];
          tmem_ld64(lane_base + TM_UV, u);
          DBG_ROW(24576, 64, u);
          tmem_ld64(lane_base + TM_OA, u);
          DBG_ROW(32768, 64, u);
        }
#endif
        st_row64_sw128(sm + Lay::WT, i, x);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      cbar();
      // ---- V'^T = U^T - S_b W^T
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          mma_bf16_ss(tm + TM_UV, sdesc_sw128(a_sb + aoff, 16, 1024),
                      sdesc_sw128(a_wt + kk * 2048, 2 * kTileBytes, 1024), ID_VP, 1);
        }
        mma_commit(mmab);
      }
      if (!wait_mma()) { aborted = true; break; }

      // ---- V'^T -> bf16 operands (plain and decayed to the chunk end);
      //      pre-decay the fp32 state by e^{gc_last}
      {
        float x[64];
        tmem_ld64(lane_base + TM_UV, x);
        DBG_ROW(40960, 64, x);
        st_row64_sw128(sm + Lay::VP, i, x);
#pragma unroll
        for (int r = 0; r < 64; ++r) x[r] *= eglv[r];
        st_row64_sw128(sm + Lay::VPD, i, x);
        const float dl = egv[63];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float t[16];
          tmem_ld16(lane_base + TM_S + 16 * q, t);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] *= dl;
          tmem_st16(lane_base + TM_S + 16 * q, t);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      cbar();
      // ---- O_b = V'^T P^T;  S += (V'^T decayed) K
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16_ss(tm + TM_OB, sdesc_sw128(a_vp + kk * 32, 16, 1024),
                      sdesc_sw128(a_p + kk * 32, 16, 1024), ID_O, kk > 0);
          mma_bf16_ss(tm + TM_S, sdesc_sw128(a_vpd + kk * 32, 16, 1024),
                      sdesc_sw128(kq + kk * 2048, 2 * kTileBytes, 1024), ID_S, 1);
        }
        mma_commit(mmab);
      }
      if (!wait_mma()) { aborted = true; break; }
      if (tid == 0) {
        mbar_arrive(&empty[s]);  // K, Q, V of this stage are no longer read
        *consumed = c + 1;
      }

      // ---- O = Diag(e^{gc}) O_a + O_b  -> bf16 staging -> TMA store
      {
        float xa[64], xb[64];
        tmem_ld64(lane_base + TM_OA, xa);
        tmem_ld64(lane_base + TM_OB, xb);
        DBG_ROW(49152, 64, xb);
        __nv_bfloat16 *stg = reinterpret_cast<__nv_bfloat16 *>(sm + Lay::AF) + (i >> 6) * 4096;
        const int col = i & 63;
#pragma unroll
        for (int r = 0; r < 64; ++r) stg[r * 64 + col] = __float2bfloat16_rn(egv[r] * xa[r] + xb[r]);
      }
      // ---- S -> S_b for the next chunk
      {
        float x[64];
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld64(lane_base + TM_S + 64 * hh, x);
          DBG_ROW(57344 + 8192 * hh, 64, x);
          st_row64_sw128(sm + Lay::SB + hh * 2 * kTileBytes, i, x);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      cbar();
      if (tid == 0) {
        tma_store_4d(&tmO, sm + Lay::AF, 0, h, t0, b);
        tma_store_4d(&tmO, sm + Lay::AF + kTileBytes, 64, h, t0, b);
        tma_store_commit();
      }
    }
    if (aborted && tid == 0) atomicOr(a.status, kStatusTimeout);

    // ---- final state
    if (!aborted && a.S_T) {
      float x[64];
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld64(lane_base + TM_S + 64 * hh, x);
        float4 *dst = reinterpret_cast<float4 *>(a.S_T + ((size_t)bh * DV + i) * DK + 64 * hh);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          dst[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
      }
    }
    if (tid == 0) tma_store_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ------------------------------------------------------------------ host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D map over a [B, T, H, d] bf16 tensor, box = 64 tokens x 64 channels.
bool make_map(CUtensorMap *m, const void *base, int B, int T, int H, int d, bool swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supports(const ChunkArgs &a) {
  return a.bf16 && !a.per_channel && a.dk == DK && a.dv == DV && a.T > 0 &&
         (size_t)a.B * a.H <= 0x7fffffffu;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream) {
  if (!chunk_tc_supports(a)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, a.q, a.B, a.T, a.H, DK, true) || !make_map(&mk, a.k, a.B, a.T, a.H, DK, true) ||
      !make_map(&mv, a.v, a.B, a.T, a.H, DV, true) || !make_map(&mo, a.o, a.B, a.T, a.H, DV, false))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gdr_chunk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  gdr_chunk_tc_kernel<<<(unsigned)((size_t)a.B * a.H), kThreads, kSmemBytes, stream>>>(mq, mk, mv,
                                                                                       mo, a);
  return cudaGetLastError();
}

}  // namespace gdr

#ifdef GDR_TC_DEBUG
extern "C" int gdr_debug_set_buffer(float *p, int chunk) {
  if (cudaMemcpyToSymbol(gdr::g_dbg, &p, sizeof p) != cudaSuccess) return 1;
  return cudaMemcpyToSymbol(gdr::g_dbg_chunk, &chunk, sizeof chunk) != cudaSuccess;
}
#endif
