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
//   Y    = (I + A)^{-1}  (16x16 diagonal blocks by forward substitution,
//                          off-diagonal blocks with mma.sync TF32)
//   T    = Y Diag(beta),  T' = T Diag(e^{gc})            -> bf16, smem
//   Q~   = Diag(e^{gc}) Q                                -> in place, smem
//   U^T  = V^T T^T,  W^T = K^T T'^T        (tcgen05, M=128 N=64 K=64)
//   V'^T = U^T + S_b (-W)^T                (tcgen05, A = S_b from TMEM)
//   O^T  = S_b Q~^T + V'^T P^T             (tcgen05, one accumulator)
//   S    = e^{gc_last} S + (V'^T Diag(e^{gc_last - gc})) K   (fp32 TMEM acc)
//
// S_b is the bf16 copy of the fp32 state, kept in TMEM as the A operand.
// e^{gc_r - gc_s} is formed as e^{gc_r} e^{-gc_s} while the chunk's total
// decay keeps e^{-gc} finite, else pairwise, so no scalar gate overflows.
//
// Warp roles (one CTA per (b, h), 320 threads):
//   warps 0-3  "state" group: V'^T -> bf16 operands, O epilogue + TMA store,
//              S -> S_b and the per-chunk state decay (TMEM lanes 0-127);
//   warps 4-7  "prep" group, one chunk ahead: gate cumsum, A/P epilogue,
//              (I + A)^{-1}, T/T', Q~, W^T -> bf16 operand;
//   warp 8     TMA producer (two input stages, no multicast) + g/beta loads;
//   warp 9     MMA issuer (one thread).
// Hand-offs are mbarriers; every wait is bounded (time-out -> device status
// word, abort flag, orderly unwind, TMEM freed).
#include <cudaTypedefs.h>

#include <mutex>

#include "gdr_internal.cuh"
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 320;
constexpr int kStages = 2;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kTileBytes = 64 * 128;    // one 64 x 64 bf16 tile
constexpr uint32_t kStageTx = 6 * kTileBytes;
constexpr float kSafeDecay = 80.f;  // e^{80} is finite in fp32

// Shared-memory layout (byte offsets from a 1024-byte aligned base).
struct Lay {
  static constexpr uint32_t KQ = 0;                             // per stage [K_h0|Q_h0|K_h1|Q_h1]
  static constexpr uint32_t V = KQ + kStages * 4 * kTileBytes;  // per stage [V_h0|V_h1]
  static constexpr uint32_t T = V + kStages * 2 * kTileBytes;   // T   K-major [r][s]
  static constexpr uint32_t TP = T + kTileBytes;                // T'  K-major [r][s]
  static constexpr uint32_t P = TP + kTileBytes;                // P   K-major [r][s], x2
  static constexpr uint32_t WT = P + 2 * kTileBytes;            // -W^T MN-major [dk][C]
  static constexpr uint32_t VP = WT + 2 * kTileBytes;           // V'^T K-major [dv][C]; O staging
  static constexpr uint32_t VPD = VP + 2 * kTileBytes;          // decayed V'^T
  static constexpr uint32_t AF = VPD + 2 * kTileBytes;          // fp32 A/Y [64][65]
  static constexpr uint32_t R = AF + 64 * 65 * 4;               // fp32 [16][49]
  static constexpr uint32_t GS = R + 16 * 49 * 4;               // per stage g[64], beta[64]
  static constexpr uint32_t VEC = GS + kStages * 512;           // x3: gc, eg, ieg, egl [64] each
  static constexpr uint32_t BAR = VEC + 3 * 1024;               // mbarriers
  static constexpr uint32_t MISC = BAR + 16 * 8;                // tmem base, abort flag, consumed
  static constexpr uint32_t END = MISC + 16;
};
static_assert(Lay::AF % 1024 == 0, "tile alignment");
constexpr size_t kSmemBytes = Lay::END + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// mbarrier slots
enum {
  B_FULL = 0,   // [2] TMA + g/beta of a stage landed          (count 1 + tx)
  B_EMPTY = 2,  // [2] stage may be refilled: MMA commit + prep  (count 2)
  B_D1F = 4,    // D1 written                                   (commit)
  B_D1E,        // D1 read by the prep group                    (128)
  B_TRDY,       // T, T', Q~, P, gate vectors of a chunk ready  (128)
  B_WTF,        // U^T, W^T written                             (commit)
  B_WTB,        // -W^T bf16 operand written                    (128)
  B_SBR,        // S_b in TMEM and the decayed S ready          (128)
  B_VPF,        // V'^T and O_a written                         (commit)
  B_VPR,        // V'^T bf16 operands written                   (128)
  B_OF,         // O and the updated S written                  (commit)
  B_FIN,        // final drain of the MMA pipe                  (commit)
  B_COUNT
};

// TMEM column map (512 allocated; 1 CTA per SM).
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_D1 = 192, TM_UV = 256, TM_WT = 320, TM_O = 384;

constexpr uint32_t ID_D1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_U = idesc_bf16(128, 64, 1, 0);
constexpr uint32_t ID_VP = idesc_bf16(128, 64, 0, 1);
constexpr uint32_t ID_O = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 1);

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&t);
}

// Write 32 fp32 values as bf16 columns [32 q, 32 q + 32) of row `row` of a
// 128B-swizzled tile whose rows are 64 bf16.
__device__ __forceinline__ void st_row32_sw128(uint8_t *tile, int row, int q, const float *x) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint4 u;
    u.x = pack_bf16(x[8 * ch + 0], x[8 * ch + 1]);
    u.y = pack_bf16(x[8 * ch + 2], x[8 * ch + 3]);
    u.z = pack_bf16(x[8 * ch + 4], x[8 * ch + 5]);
    u.w = pack_bf16(x[8 * ch + 6], x[8 * ch + 7]);
    *reinterpret_cast<uint4 *>(tile + sw128_off(row, 32 * q + 8 * ch)) = u;
  }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  float a[16], b[16];
  tmem_ld16(taddr, a);
  tmem_ld16(taddr + 16, b);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    v[e] = a[e];
    v[16 + e] = b[e];
  }
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Barrier over one 128-thread group that also ORs a predicate.
__device__ __forceinline__ bool group_any(uint32_t bar_id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(bar_id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void group_bar(uint32_t bar_id) { named_bar_sync(bar_id, 128); }

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
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

// (I + A)^{-1} in place for a strictly lower 64x64 fp32 matrix (row stride
// 65) with one 128-thread group (local thread id t, warp w = t / 32):
// diagonal 16x16 blocks by forward substitution (warp w owns block w), then
// for block rows b = 1..3: R_b = sum_{k<b} A_bk Y_k and Y_b = -D_bb R_b,
// 8-column tiles on mma.sync (TF32 operands rounded to nearest).
__device__ void invert_unit_lower(float *AF, float *R, int t, uint32_t bar_id) {
  const int warp = t >> 5, lane = t & 31;
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
  group_bar(bar_id);
  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int b = 1; b < 4; ++b) {
    const int ntiles = 2 * b;
    for (int nt = warp; nt < ntiles; nt += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = nt >> 1; k < b; ++k) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const int col = 16 * k + 8 * ks;
          uint32_t af[4], bf[2];
          af[0] = to_tf32(AF[(16 * b + g) * 65 + col + tq]);
          af[1] = to_tf32(AF[(16 * b + g + 8) * 65 + col + tq]);
          af[2] = to_tf32(AF[(16 * b + g) * 65 + col + tq + 4]);
          af[3] = to_tf32(AF[(16 * b + g + 8) * 65 + col + tq + 4]);
          bf[0] = to_tf32(AF[(col + tq) * 65 + 8 * nt + g]);
          bf[1] = to_tf32(AF[(col + tq + 4) * 65 + 8 * nt + g]);
          mma_tf32_16x8x8(acc, af, bf);
        }
      }
      R[g * 49 + 8 * nt + 2 * tq] = acc[0];
      R[g * 49 + 8 * nt + 2 * tq + 1] = acc[1];
      R[(g + 8) * 49 + 8 * nt + 2 * tq] = acc[2];
      R[(g + 8) * 49 + 8 * nt + 2 * tq + 1] = acc[3];
    }
    group_bar(bar_id);
    for (int nt = warp; nt < ntiles; nt += 4) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const int col = 16 * b + 8 * ks;
        uint32_t af[4], bf[2];
        af[0] = to_tf32(AF[(16 * b + g) * 65 + col + tq]);
        af[1] = to_tf32(AF[(16 * b + g + 8) * 65 + col + tq]);
        af[2] = to_tf32(AF[(16 * b + g) * 65 + col + tq + 4]);
        af[3] = to_tf32(AF[(16 * b + g + 8) * 65 + col + tq + 4]);
        bf[0] = to_tf32(R[(8 * ks + tq) * 49 + 8 * nt + g]);
        bf[1] = to_tf32(R[(8 * ks + tq + 4) * 49 + 8 * nt + g]);
        mma_tf32_16x8x8(acc, af, bf);
      }
      AF[(16 * b + g) * 65 + 8 * nt + 2 * tq] = -acc[0];
      AF[(16 * b + g) * 65 + 8 * nt + 2 * tq + 1] = -acc[1];
      AF[(16 * b + g + 8) * 65 + 8 * nt + 2 * tq] = -acc[2];
      AF[(16 * b + g + 8) * 65 + 8 * nt + 2 * tq + 1] = -acc[3];
    }
    group_bar(bar_id);
  }
}

#ifdef GDR_TC_DEBUG
// Debug build only: stage values of one chunk of CTA 0 are copied out.
__device__ float *g_dbg = nullptr;
__device__ int g_dbg_chunk = 0;
#define DBG_ROW(off, ncol, src)                                                       \
  do {                                                                                \
    if (g_dbg && blockIdx.x == 0 && c == g_dbg_chunk)                                \
      for (int _e = 0; _e < 32; ++_e) g_dbg[(off) + lrow * (ncol) + _e] = (src)[_e]; \
  } while (0)
#else
#define DBG_ROW(off, ncol, src) \
  do {                          \
  } while (0)
#endif

// 10 warps leave three warps on some SM sub-partitions, whose register file
// is a quarter of the SM's: the launch bound caps registers accordingly.
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
  const int n = (T + C - 1) / C;

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lay::MISC + 4);
  volatile int *consumed = reinterpret_cast<volatile int *>(sm + Lay::MISC + 8);
  float *AF = reinterpret_cast<float *>(sm + Lay::AF);
  float *Rs = reinterpret_cast<float *>(sm + Lay::R);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_FULL + s], 1);
      mbar_init(&bars[B_EMPTY + s], 2);
    }
    mbar_init(&bars[B_D1F], 1);
    mbar_init(&bars[B_D1E], 128);
    mbar_init(&bars[B_TRDY], 128);
    mbar_init(&bars[B_WTF], 1);
    mbar_init(&bars[B_WTB], 128);
    mbar_init(&bars[B_SBR], 128);
    mbar_init(&bars[B_VPF], 1);
    mbar_init(&bars[B_VPR], 128);
    mbar_init(&bars[B_OF], 1);
    mbar_init(&bars[B_FIN], 1);
    *abort_flag = 0;
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
  const uint32_t lane_base = tm + ((uint32_t)((warp & 3) * 32) << 16);

  if (warp == 8) {
    // ================================================================ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int issued = 0;
    for (int c = 0; c < n; ++c) {
      const int s = c & 1;
      if (c >= kStages) {
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(&bars[B_EMPTY + s], ((c >> 1) - 1) & 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
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
        uint64_t *fb = &bars[B_FULL + s];
        mbar_arrive_expect_tx(fb, kStageTx);
        uint8_t *kq = sm + Lay::KQ + s * 4 * kTileBytes;
        uint8_t *vv = sm + Lay::V + s * 2 * kTileBytes;
        tma_load_4d(kq + 0 * kTileBytes, &tmK, fb, 0, h, t0, b);
        tma_load_4d(kq + 1 * kTileBytes, &tmQ, fb, 0, h, t0, b);
        tma_load_4d(kq + 2 * kTileBytes, &tmK, fb, 64, h, t0, b);
        tma_load_4d(kq + 3 * kTileBytes, &tmQ, fb, 64, h, t0, b);
        tma_load_4d(vv + 0 * kTileBytes, &tmV, fb, 0, h, t0, b);
        tma_load_4d(vv + 1 * kTileBytes, &tmV, fb, 64, h, t0, b);
      }
      ++issued;
    }
    // Loads issued but never consumed exist only after an abort: let them land.
    if (lane == 0) {
      for (int c = *consumed; c < issued; ++c)
        mbar_wait_bounded(&bars[B_FULL + (c & 1)], (c >> 1) & 1, kWaitNs);
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t a_kq = smem_u32(sm + Lay::KQ), a_v = smem_u32(sm + Lay::V);
      const uint32_t a_t = smem_u32(sm + Lay::T), a_tp = smem_u32(sm + Lay::TP);
      const uint32_t a_p = smem_u32(sm + Lay::P), a_wt = smem_u32(sm + Lay::WT);
      const uint32_t a_vp = smem_u32(sm + Lay::VP), a_vpd = smem_u32(sm + Lay::VPD);
      auto W = [&](int slot, uint32_t parity) {
        const bool ok = wait_or_abort(&bars[slot], parity, abort_flag);
        tc_fence_after();
        return ok;
      };
      auto issue_d1 = [&](int c) {  // D1 = [K; Q] K^T
        const uint32_t kq = a_kq + (c & 1) * 4 * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          mma_bf16_ss(tm + TM_D1, sdesc_sw128(kq + off, 16, 1024),
                      sdesc_sw128(kq + off, 16, 1024), ID_D1, kk > 0);
        }
        mma_commit(&bars[B_D1F]);
      };
      auto issue_uw = [&](int c) {  // U^T = V^T T^T, W^T = K^T T'^T
        const uint32_t kq = a_kq + (c & 1) * 4 * kTileBytes;
        const uint32_t vv = a_v + (c & 1) * 2 * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16_ss(tm + TM_UV, sdesc_sw128(vv + kk * 2048, kTileBytes, 1024),
                      sdesc_sw128(a_t + kk * 32, 16, 1024), ID_U, kk > 0);
          mma_bf16_ss(tm + TM_WT, sdesc_sw128(kq + kk * 2048, 2 * kTileBytes, 1024),
                      sdesc_sw128(a_tp + kk * 32, 16, 1024), ID_U, kk > 0);
        }
        mma_commit(&bars[B_WTF]);
      };
      bool ok = true;
      do {
        if (!(ok = W(B_FULL, 0))) break;
        issue_d1(0);
        if (!(ok = W(B_TRDY, 0))) break;
        issue_uw(0);
        // Each barrier below completes once per chunk and is waited on by
        // parity, so no producer may run two phases ahead of a waiter.  D1 of
        // chunk c+1 is issued only after S_b of chunk c is ready, i.e. after
        // the state group has consumed the gate vectors of chunk c; this
        // bounds the prep group's lead to one chunk.
        for (int c = 0; c < n && ok; ++c) {
          const uint32_t ph = c & 1;
          const uint32_t kq = a_kq + (c & 1) * 4 * kTileBytes;
          // V'^T = U^T + S_b (-W)^T ;  O = S_b Q~^T
          if (!(ok = W(B_WTB, ph) && W(B_SBR, ph))) break;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_bf16_ts(tm + TM_UV, tm + TM_SB + 8 * kk,
                        sdesc_sw128(a_wt + kk * 2048, 2 * kTileBytes, 1024), ID_VP, 1);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t boff = kTileBytes + (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
            mma_bf16_ts(tm + TM_O, tm + TM_SB + 8 * kk, sdesc_sw128(kq + boff, 16, 1024), ID_O,
                        kk > 0);
          }
          mma_commit(&bars[B_VPF]);
          if (c + 1 < n) {
            if (!(ok = W(B_D1E, ph) && W(B_FULL + ((c + 1) & 1), ((c + 1) >> 1) & 1))) break;
            issue_d1(c + 1);
          }
          // O += V'^T P^T ;  S += (V'^T decayed) K
          if (!(ok = W(B_VPR, ph))) break;
          const uint32_t pp = a_p + (c & 1) * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tm + TM_O, sdesc_sw128(a_vp + kk * 32, 16, 1024),
                        sdesc_sw128(pp + kk * 32, 16, 1024), ID_O, 1);
            mma_bf16_ss(tm + TM_S, sdesc_sw128(a_vpd + kk * 32, 16, 1024),
                        sdesc_sw128(kq + kk * 2048, 2 * kTileBytes, 1024), ID_S, 1);
          }
          mma_commit(&bars[B_OF]);
          mma_commit(&bars[B_EMPTY + (c & 1)]);
          *consumed = c + 1;
          if (c + 1 < n) {
            if (!(ok = W(B_TRDY, (c + 1) & 1))) break;
            issue_uw(c + 1);
          }
        }
      } while (0);
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(&bars[B_FIN]);
      mbar_wait_bounded(&bars[B_FIN], 0, kWaitNs);
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp >= 4) {
    // ================================================================ prep group
    const int t = tid - 128;  // 0..127, also the TMEM lane
    const int lrow = t;
    (void)lrow;
    constexpr uint32_t kBar = 3;
    for (int c = 0; c < n; ++c) {
      const int s = c & 1;
      const uint32_t ph = c & 1;
      float *vec = reinterpret_cast<float *>(sm + Lay::VEC + (c % 3) * 1024);
      float *gcv = vec, *egv = vec + 64, *iegv = vec + 128, *eglv = vec + 192;
      if (group_any(kBar, !wait_or_abort(&bars[B_FULL + s], (c >> 1) & 1, abort_flag))) break;
      const float *gs = reinterpret_cast<const float *>(sm + Lay::GS + s * 512);
      const float *bs = gs + 64;
      if (warp == 4) {  // cumulative log decay and the derived factors
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
        iegv[lane] = __expf(-x0);
        iegv[lane + 32] = __expf(-x1);
        eglv[lane] = __expf(gl - x0);
        eglv[lane + 32] = __expf(gl - x1);
      }
      group_bar(kBar);
      const bool factored = -gcv[63] < kSafeDecay;
      // ---- A (lanes 0-63) and P (lanes 64-127) from D1
      if (group_any(kBar, !wait_or_abort(&bars[B_D1F], ph, abort_flag))) break;
      tc_fence_after();
      {
        const int r = t & 63;
        const float gr = gcv[r];
        const float br = t < 64 ? bs[r] : 1.f;
        const float fr = br * egv[r];
        uint8_t *ptile = sm + Lay::P + s * kTileBytes;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_D1 + 32 * q, x);
          DBG_ROW(32 * q, 64, x);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int s2 = 32 * q + e;
            const float d = factored ? fr * iegv[s2] : br * __expf(gr - gcv[s2]);
            x[e] = (t < 64 ? (s2 < r) : (s2 <= r)) ? x[e] * d : 0.f;
          }
          if (t < 64) {
#pragma unroll
            for (int e = 0; e < 32; ++e) AF[r * 65 + 32 * q + e] = x[e];
          } else {
            st_row32_sw128(ptile, r, q, x);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[B_D1E]);
      group_bar(kBar);
      // ---- Y = (I + A)^{-1}
      invert_unit_lower(AF, Rs, t, kBar);
#ifdef GDR_TC_DEBUG
      if (t < 64) {
        DBG_ROW(12288, 64, AF + t * 65);
        DBG_ROW(12288 + 32, 64, AF + t * 65 + 32);
      }
#endif
      // ---- T (lanes 0-63) and T' (lanes 64-127) as bf16 operands
      {
        const int r = t & 63;
        uint8_t *tile = sm + (t < 64 ? Lay::T : Lay::TP);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int s2 = 32 * q + e;
            x[e] = AF[r * 65 + s2] * bs[s2] * (t < 64 ? 1.f : egv[s2]);
          }
          st_row32_sw128(tile, r, q, x);
        }
      }
      // ---- Q~ = Diag(e^{gc}) Q in place (both 64-column halves)
      {
        uint8_t *kq = sm + Lay::KQ + s * 4 * kTileBytes;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int idx = t + 128 * m;  // 16-byte chunk index over 2 x 64 rows x 8
          const int half = idx >> 9, row = (idx >> 3) & 63, ch = idx & 7;
          uint4 *p = reinterpret_cast<uint4 *>(kq + kTileBytes + half * 2 * kTileBytes +
                                               row * 128 + ch * 16);
          uint4 u = *p;
          const float e = egv[row];
          uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 v2 = *reinterpret_cast<__nv_bfloat162 *>(&w[j]);
            float2 f = __bfloat1622float2(v2);
            w[j] = pack_bf16(f.x * e, f.y * e);
          }
          *p = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_TRDY]);
      group_bar(kBar);
      if (t == 0) mbar_arrive(&bars[B_EMPTY + s]);  // g, beta of this stage no longer read
      // ---- -W^T -> bf16 MN-major operand (row j = this thread's lane)
      if (group_any(kBar, !wait_or_abort(&bars[B_WTF], ph, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float x[32];
        tmem_ld32(lane_base + TM_WT + 32 * q, x);
        DBG_ROW(16384 + 32 * q, 64, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = -x[e];
        st_row32_sw128(sm + Lay::WT, t, q, x);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_WTB]);
    }
  } else {
    // ================================================================ state group
    const int i = tid;  // TMEM lane = value channel
    const int lrow = i;
    (void)lrow;
    constexpr uint32_t kBar = 2;
    bool ok = true;
    // Initial state: S = S0 e^{gc_last(0)} (fp32), S_b = bf16(S0).
    if (group_any(kBar, !wait_or_abort(&bars[B_TRDY], 0, abort_flag))) ok = false;
    if (ok) {
      const float *vec = reinterpret_cast<const float *>(sm + Lay::VEC);
      const float dl = vec[64 + 63];  // e^{gc_last} of chunk 0
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          x[e] = a.S0 ? a.S0[((size_t)bh * DV + i) * DK + 32 * q + e] : 0.f;
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        tmem_st16u(lane_base + TM_SB + 16 * q, u);
        float y0[16], y1[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          y0[e] = x[e] * dl;
          y1[e] = x[16 + e] * dl;
        }
        tmem_st16(lane_base + TM_S + 32 * q, y0);
        tmem_st16(lane_base + TM_S + 32 * q + 16, y1);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_SBR]);
    }
    for (int c = 0; ok && c < n; ++c) {
      const uint32_t ph = c & 1;
      const float *vec = reinterpret_cast<const float *>(sm + Lay::VEC + (c % 3) * 1024);
      const float *eglv = vec + 192;
      // ---- V'^T -> bf16 operands (plain and decayed to the chunk end)
      if (group_any(kBar, !wait_or_abort(&bars[B_VPF], ph, abort_flag))) { ok = false; break; }
      tc_fence_after();
      if (i == 0) tma_store_wait_read0();  // previous O staging (aliases VP) is free
      group_bar(kBar);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float x[32];
        tmem_ld32(lane_base + TM_UV + 32 * q, x);
        DBG_ROW(40960 + 32 * q, 64, x);
        st_row32_sw128(sm + Lay::VP, i, q, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= eglv[32 * q + e];
        st_row32_sw128(sm + Lay::VPD, i, q, x);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_VPR]);
      // ---- O -> bf16 -> staging (VP region) -> TMA store
      if (group_any(kBar, !wait_or_abort(&bars[B_OF], ph, abort_flag))) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t *stg = reinterpret_cast<uint32_t *>(sm + Lay::VP + (i >> 6) * kTileBytes);
        const int col = i & 63;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_O + 32 * q, x);
          DBG_ROW(49152 + 32 * q, 64, x);
          // lanes i, i^1 swap so each writes two adjacent channels of one token
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float lo = x[2 * e], hi = x[2 * e + 1];  // tokens 32q+2e, +1
            const float send = (i & 1) ? lo : hi;
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            const int r = 32 * q + 2 * e + (i & 1);
            const uint32_t w = (i & 1) ? pack_bf16(recv, hi) : pack_bf16(lo, recv);
            stg[(r * 64 + (col & ~1)) >> 1] = w;
          }
        }
      }
      fence_proxy_async_smem();
      group_bar(kBar);
      if (i == 0) {
        tma_store_4d(&tmO, sm + Lay::VP, 0, h, c * C, b);
        tma_store_4d(&tmO, sm + Lay::VP + kTileBytes, 64, h, c * C, b);
        tma_store_commit();
      }
      if (c + 1 < n) {
        // ---- S (= state after this chunk) -> S_b; pre-decay by the next chunk
        if (group_any(kBar, !wait_or_abort(&bars[B_TRDY], (c + 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        const float *vn = reinterpret_cast<const float *>(sm + Lay::VEC + ((c + 1) % 3) * 1024);
        const float dl = vn[64 + 63];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          DBG_ROW(57344 + 32 * q, 128, x);
          uint32_t u[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
          tmem_st16u(lane_base + TM_SB + 16 * q, u);
          float y0[16], y1[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            y0[e] = x[e] * dl;
            y1[e] = x[16 + e] * dl;
          }
          tmem_st16(lane_base + TM_S + 32 * q, y0);
          tmem_st16(lane_base + TM_S + 32 * q + 16, y1);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[B_SBR]);
      } else if (a.S_T) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          DBG_ROW(57344 + 32 * q, 128, x);
          float4 *dst = reinterpret_cast<float4 *>(a.S_T + ((size_t)bh * DV + i) * DK + 32 * q);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        }
      }
    }
    if (i == 0) tma_store_wait0();
    if (!ok && i == 0) atomicOr(a.status, kStatusTimeout);
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
