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
//   U^T  = V^T T^T,  W^T = K^T T'^T        (tcgen05, M=128 N=64 K=64)
//   V'^T = U^T + S_b (-W)^T                (tcgen05, A = S_b from TMEM)
//   O^T  = (S_b Q^T) Diag(e^{gc}) + V'^T P^T   (tcgen05, two accumulators)
//   S    = e^{gc_last} S + (V'^T Diag(e^{gc_last - gc})) K   (fp32 TMEM acc)
//
// S_b is the bf16 copy of the fp32 state, kept in TMEM as the A operand.
// e^{gc_r - gc_s} is formed as e^{gc_r} e^{-gc_s} while the chunk's total
// decay keeps e^{-gc} finite, else pairwise, so no scalar gate overflows.
//
// Warp roles (one CTA per (b, h), 320 threads):
//   warps 0-3  "state" group: V'^T -> bf16 operands, O epilogue (direct stores),
//              S -> S_b and the per-chunk state decay (TMEM lanes 0-127);
//   warps 4-7  "prep" group, one chunk ahead: gate cumsum, A/P epilogue,
//              (I + A)^{-1}, T/T', W^T -> bf16 operand;
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
constexpr int kPrepWarps = 4;
constexpr int kPrepThreads = 32 * kPrepWarps;
constexpr int kThreads = 320;  // 4 state + 4 prep + producer + MMA warps
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kStages = 2;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kTileBytes = 64 * 128;    // one 64 x 64 bf16 tile
constexpr uint32_t kStageTx = 6 * kTileBytes;
constexpr float kSafeDecay = 80.f;  // e^{80} is finite in fp32
// Row stride (floats) of the fp32 A/Y matrix: rows stay 16-byte aligned, and
// mma.sync A-fragment loads hit distinct banks.
constexpr int LDA = 68;

// Shared-memory layout (byte offsets from a 1024-byte aligned base).
struct Lay {
  static constexpr uint32_t KQ = 0;                             // per stage [K_h0|Q_h0|K_h1|Q_h1]
  static constexpr uint32_t V = KQ + kStages * 4 * kTileBytes;  // per stage [V_h0|V_h1]
  static constexpr uint32_t T = V + kStages * 2 * kTileBytes;   // T   K-major [r][s]
  static constexpr uint32_t TP = T + kTileBytes;                // T'  K-major [r][s]
  static constexpr uint32_t P = TP + kTileBytes;                // P   K-major [r][s], x2
  static constexpr uint32_t WT = P + 2 * kTileBytes;            // -W^T MN-major [dk][C]
  static constexpr uint32_t VP = WT + 2 * kTileBytes;           // V'^T K-major [dv][C]
  static constexpr uint32_t VPD = VP + 2 * kTileBytes;          // decayed V'^T
  static constexpr uint32_t AF = VPD + 2 * kTileBytes;          // fp32 A, then Y [64][LDA]
  static constexpr uint32_t SCR = AF + 64 * LDA * 4;            // fp32 inverse scratch 4 x [16][8]
  static constexpr uint32_t GS = SCR + 4 * 128 * 4;             // per stage g[64], beta[64]
  static constexpr uint32_t VEC = GS + kStages * 512;           // x3: gc, eg, ieg, egl [64] each
  static constexpr uint32_t SVEC = VEC + 3 * 1024;              // x2: eg, egl [64] (state group)
  static constexpr uint32_t BAR = SVEC + 2 * 512;               // mbarriers
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
  B_D1E,        // D1 read by the prep group                    (256)
  B_TRDY,       // T, T', P, gate vectors of a chunk ready      (256)
  B_WTF,        // U^T, W^T written                             (commit)
  B_WTB,        // -W^T bf16 operand written                    (256)
  B_SBR,        // S_b in TMEM and the decayed S ready          (128)
  B_VPF,        // V'^T and O_a written                         (commit)
  B_VPR,        // V'^T bf16 operands written                   (128)
  B_SF,         // the updated S written                        (commit)
  B_OF,         // O_a and O_b written                          (commit)
  B_FIN,        // final drain of the MMA pipe                  (commit)
  B_COUNT
};

// TMEM column map (512 allocated; 1 CTA per SM).
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_D1 = 192, TM_UV = 256, TM_WT = 320, TM_O = 384,
                   TM_OA = 448;

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

// 64 consecutive TMEM columns of this thread's lane: four loads, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  float a0[16], a1[16], a2[16], a3[16];
  tmem_ld16(taddr, a0);
  tmem_ld16(taddr + 16, a1);
  tmem_ld16(taddr + 32, a2);
  tmem_ld16(taddr + 48, a3);
  tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    v[e] = a0[e];
    v[16 + e] = a1[e];
    v[32 + e] = a2[e];
    v[48 + e] = a3[e];
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

// Warp-group barriers: id 2 = state group (128 threads), id 3 = prep group
// (kPrepThreads).
__device__ __forceinline__ uint32_t group_threads(uint32_t bar_id) {
  return bar_id == 3 ? (uint32_t)kPrepThreads : 128u;
}

// Barrier over one warp group that also ORs a predicate.
__device__ __forceinline__ bool group_any(uint32_t bar_id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(bar_id), "r"(group_threads(bar_id))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void group_bar(uint32_t bar_id) {
  named_bar_sync(bar_id, group_threads(bar_id));
}

// Bounded wait that also gives up as soon as another role has aborted.
// The thread sleeps inside try_wait (suspend hint) between checks.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, 20000)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Group-wide wait: lane 0 of each warp polls, the warp shares its result,
// and the group agrees (any failure -> every thread sees failure).
__device__ __forceinline__ bool group_wait(uint32_t bar_id, uint64_t *bar, uint32_t parity,
                                           volatile int *abort_flag, int lane) {
  bool ok = true;
  if (lane == 0) ok = wait_or_abort(bar, parity, abort_flag);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return !group_any(bar_id, !ok);
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

// Helpers of the blocked inverse below (one warp, mma.sync m16n8k8 TF32
// fragments: g = lane / 4, tq = lane % 4).
struct Frag {
  int g, tq;
  float *scr;  // warp-private [16][8] fp32 scratch
  // A fragment of the 16x8 block of AF at (row0, col0).
  __device__ __forceinline__ void a(const float *AF, int row0, int col0, uint32_t (&af)[4]) const {
    af[0] = to_tf32(AF[(row0 + g) * LDA + col0 + tq]);
    af[1] = to_tf32(AF[(row0 + g + 8) * LDA + col0 + tq]);
    af[2] = to_tf32(AF[(row0 + g) * LDA + col0 + tq + 4]);
    af[3] = to_tf32(AF[(row0 + g + 8) * LDA + col0 + tq + 4]);
  }
  // 16x8 accumulator fragment -> B fragments of two k-steps (rows 0-7, 8-15).
  __device__ __forceinline__ void to_b(const float (&cf)[4], uint32_t (&bf)[2][2]) const {
    scr[g * 8 + 2 * tq] = cf[0];
    scr[g * 8 + 2 * tq + 1] = cf[1];
    scr[(g + 8) * 8 + 2 * tq] = cf[2];
    scr[(g + 8) * 8 + 2 * tq + 1] = cf[3];
    __syncwarp();
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      bf[ks][0] = to_tf32(scr[(8 * ks + tq) * 8 + g]);
      bf[ks][1] = to_tf32(scr[(8 * ks + tq + 4) * 8 + g]);
    }
    __syncwarp();
  }
};

// One 8-column strip (first column `col`) of column block J of Y = (I + A)^{-1}:
// Y_JJ = D_JJ (already in AF), Y_bJ = -D_bb sum_{k=J}^{b-1} A_bk Y_kJ for
// b > J, swept down the block rows; the finished blocks stay in `yout[b]`.
// J is a template parameter so that every loop is fully static.
template <int J>
__device__ __forceinline__ void inverse_strip(const float *AF, const Frag &f, int col,
                                              float (&yout)[4][4]) {
  uint32_t yb[4][2][2];
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    yb[J][ks][0] = to_tf32(AF[(16 * J + 8 * ks + f.tq) * LDA + col + f.g]);
    yb[J][ks][1] = to_tf32(AF[(16 * J + 8 * ks + f.tq + 4) * LDA + col + f.g]);
  }
#pragma unroll
  for (int bb = J + 1; bb < 4; ++bb) {
    float racc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = J; k < bb; ++k) {
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t af[4];
        f.a(AF, 16 * bb, 16 * k + 8 * ks, af);
        mma_tf32_16x8x8(racc, af, yb[k][ks]);
      }
    }
    uint32_t rb[2][2];
    f.to_b(racc, rb);
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t af[4];
      f.a(AF, 16 * bb, 16 * bb + 8 * ks, af);
      mma_tf32_16x8x8(yacc, af, rb[ks]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) yout[bb][e] = -yacc[e];
    if (bb < 3) f.to_b(yout[bb], yb[bb]);
  }
}

template <int J>
__device__ __forceinline__ void store_strip(float *AF, const Frag &f, int col,
                                            const float (&yout)[4][4]) {
#pragma unroll
  for (int bb = J + 1; bb < 4; ++bb) {
    AF[(16 * bb + f.g) * LDA + col + 2 * f.tq] = yout[bb][0];
    AF[(16 * bb + f.g) * LDA + col + 2 * f.tq + 1] = yout[bb][1];
    AF[(16 * bb + f.g + 8) * LDA + col + 2 * f.tq] = yout[bb][2];
    AF[(16 * bb + f.g + 8) * LDA + col + 2 * f.tq + 1] = yout[bb][3];
  }
}

// (I + A)^{-1} in place for a strictly lower 64x64 fp32 matrix A (row stride
// LDA, zero above the diagonal blocks) with the 4-warp prep group (local
// thread t, warp w = t / 32), in 16x16 blocks:
//  1. diagonal blocks D_bb = (I + A_bb)^{-1} by forward substitution (warp b);
//  2. every 8-column strip of a column block is independent, so each warp
//     sweeps its strips down the block rows with mma.sync (TF32 operands
//     rounded to nearest, fp32 accumulation);
//  3. after a group barrier the off-diagonal blocks overwrite A.
// Strips (column block j, half hf): warp 0 -> (0,0); warp 1 -> (0,1);
// warp 2 -> (1,0), (2,0); warp 3 -> (1,1), (2,1).  (The measured in-kernel
// time of this form beat an fp32 CUDA-core strip sweep, although mma.sync
// queues behind concurrent tcgen05 work.)
__device__ void invert_unit_lower(float *AF, float *R, int t, uint32_t bar_id) {
  const int warp = t >> 5, lane = t & 31;
  {
    const int w = warp, c = lane & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
    const float *Ab = AF + (16 * w) * LDA + 16 * w;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < (i + 3) / 4; ++k4) {
        const float4 av = *reinterpret_cast<const float4 *>(Ab + i * LDA + 4 * k4);
        if (4 * k4 + 0 < i) acc += av.x * x[4 * k4 + 0];
        if (4 * k4 + 1 < i) acc += av.y * x[4 * k4 + 1];
        if (4 * k4 + 2 < i) acc += av.z * x[4 * k4 + 2];
        if (4 * k4 + 3 < i) acc += av.w * x[4 * k4 + 3];
      }
      x[i] = (i > c) ? -acc : x[i];
    }
    __syncwarp();
    if (lane < 16) {
      float *Yb = AF + (16 * w) * LDA + 16 * w;
#pragma unroll
      for (int i = 0; i < 16; ++i) Yb[i * LDA + c] = x[i];
    }
  }
  group_bar(bar_id);
  const Frag f{lane >> 2, lane & 3, R + warp * 128};
  const int hf = warp & 1;
  float y0[4][4], y1[4][4];
  if (warp < 2) {
    inverse_strip<0>(AF, f, 8 * hf, y0);
  } else {
    inverse_strip<1>(AF, f, 16 + 8 * hf, y0);
    inverse_strip<2>(AF, f, 32 + 8 * hf, y1);
  }
  group_bar(bar_id);  // every read of A is done: store the off-diagonal blocks
  if (warp < 2) {
    store_strip<0>(AF, f, 8 * hf, y0);
  } else {
    store_strip<1>(AF, f, 16 + 8 * hf, y0);
    store_strip<2>(AF, f, 32 + 8 * hf, y1);
  }
  group_bar(bar_id);
}

// One warp: cumulative log decay of a chunk (g[64] -> gc[64] in log space,
// inclusive prefix sum) held as lanes r and r + 32; returns the chunk total.
__device__ __forceinline__ float chunk_cumsum(const float *g, int lane, float &x0, float &x1) {
  x0 = g[lane];
  x1 = g[lane + 32];
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
  return __shfl_sync(0xffffffffu, x1, 31);
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

// Each SM sub-partition holds a quarter of the register file and up to three
// of the block's ten warps: the launch bound caps registers at 168.
__global__ void __launch_bounds__(kThreads, 1)
    gdr_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, ChunkArgs a) {
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

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_FULL + s], 1);
      mbar_init(&bars[B_EMPTY + s], 2);
    }
    mbar_init(&bars[B_D1F], 1);
    mbar_init(&bars[B_D1E], kPrepThreads);
    mbar_init(&bars[B_TRDY], kPrepThreads);
    mbar_init(&bars[B_WTF], 1);
    mbar_init(&bars[B_WTB], kPrepThreads);
    mbar_init(&bars[B_SBR], 128);
    mbar_init(&bars[B_VPF], 1);
    mbar_init(&bars[B_VPR], 128);
    mbar_init(&bars[B_SF], 1);
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

  if (warp == kProducerWarp) {
    // ================================================================ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int last_issued[kStages] = {-1, -1};  // latest chunk loaded into each stage
    for (int c = 0; c < n; ++c) {
      const int s = c & 1;
      if (c >= kStages) {
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(&bars[B_EMPTY + s], ((c >> 1) - 1) & 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      // Testing hook: this chunk's load is never issued, so its consumers'
      // bounded waits run out and the kernel unwinds (no trap, no hang).
      if (c == a.skip_stage_chunk) continue;
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
      last_issued[s] = c;
    }
    // A load issued but never consumed exists only after an abort: let it land
    // before the CTA exits.
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        const int c = last_issued[s];
        if (c >= 0 && c >= *consumed)
          mbar_wait_bounded(&bars[B_FULL + s], (c >> 1) & 1, kWaitNs);
      }
    }
  } else if (warp == kMmaWarp) {
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
        if (n > 1) {
          if (!(ok = W(B_D1E, 0) && W(B_FULL + 1, 0))) break;
          issue_d1(1);
        }
        // Each barrier completes once per chunk and is waited on by parity,
        // so no arrival may run two phases ahead of its waiter: every
        // producer of a phase first waits, directly or through this thread's
        // program order, for its consumer's previous phase.
        for (int c = 0; c < n && ok; ++c) {
          const uint32_t ph = c & 1;
          const uint32_t kq = a_kq + (c & 1) * 4 * kTileBytes;
          // V'^T = U^T + S_b (-W)^T
          if (!(ok = W(B_WTB, ph) && W(B_SBR, ph))) break;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            mma_bf16_ts(tm + TM_UV, tm + TM_SB + 8 * kk,
                        sdesc_sw128(a_wt + kk * 2048, 2 * kTileBytes, 1024), ID_VP, 1);
          }
          mma_commit(&bars[B_VPF]);
          // O_a = S_b Q^T ;  S += (V'^T decayed) K ;  O_b = V'^T P^T.  O_a is
          // issued before the SF commit: SF then also covers the last read
          // of S_b, which the state group overwrites once SF completes.
          if (!(ok = W(B_VPR, ph))) break;
          const uint32_t pp = a_p + (c & 1) * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t boff = kTileBytes + (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
            mma_bf16_ts(tm + TM_OA, tm + TM_SB + 8 * kk, sdesc_sw128(kq + boff, 16, 1024), ID_O,
                        kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tm + TM_S, sdesc_sw128(a_vpd + kk * 32, 16, 1024),
                        sdesc_sw128(kq + kk * 2048, 2 * kTileBytes, 1024), ID_S, 1);
          }
          mma_commit(&bars[B_SF]);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tm + TM_O, sdesc_sw128(a_vp + kk * 32, 16, 1024),
                        sdesc_sw128(pp + kk * 32, 16, 1024), ID_O, kk > 0);
          }
          mma_commit(&bars[B_OF]);
          mma_commit(&bars[B_EMPTY + (c & 1)]);
          *consumed = c + 1;
          if (c + 1 < n) {
            if (!(ok = W(B_TRDY, (c + 1) & 1))) break;
            issue_uw(c + 1);
          }
          if (c + 2 < n) {
            if (!(ok = W(B_D1E, (c + 1) & 1) && W(B_FULL + (c & 1), ((c + 2) >> 1) & 1))) break;
            issue_d1(c + 2);
          }
        }
      } while (0);
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(&bars[B_FIN]);
      mbar_wait_bounded(&bars[B_FIN], 0, kWaitNs);
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp >= 4 && warp < 4 + kPrepWarps) {
    // ================================================================ prep group
    // TMEM lane rl = pt; each thread handles both 32-column halves hp of
    // its 64-column rows.
    const int pt = tid - 128, rl = pt & 127, hp0 = 0, pw = pt >> 5;
    constexpr int kHalfStep = 1;
    const int lrow = rl;
    (void)lrow;
    constexpr uint32_t kBar = 3;
    for (int c = 0; c < n; ++c) {
      const int s = c & 1;
      const uint32_t ph = c & 1;
      float *vec = reinterpret_cast<float *>(sm + Lay::VEC + (c % 3) * 1024);
      float *gcv = vec, *egv = vec + 64, *iegv = vec + 128, *eglv = vec + 192;
      if (!group_wait(kBar, &bars[B_FULL + s], (c >> 1) & 1, abort_flag, lane)) break;
      const float *gs = reinterpret_cast<const float *>(sm + Lay::GS + s * 512);
      const float *bs = gs + 64;
      if (pw == 0) {  // cumulative log decay and the derived factors
        float x0, x1;
        const float gl = chunk_cumsum(gs, lane, x0, x1);
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
      // ---- A (lanes 0-63) and P (lanes 64-127) from D1, 32 columns each
      if (!group_wait(kBar, &bars[B_D1F], ph, abort_flag, lane)) break;
      tc_fence_after();
      for (int hp = hp0; hp < 2; hp += kHalfStep) {
        const int r = rl & 63;
        const float gr = gcv[r];
        const float br = rl < 64 ? bs[r] : 1.f;
        const float fr = br * egv[r];
        float x[32];
        tmem_ld32(lane_base + TM_D1 + 32 * hp, x);
        DBG_ROW(32 * hp, 64, x);
        const int lim = (rl < 64 ? r : r + 1) - 32 * hp;  // A: s < r, P: s <= r
        // The decay form is chosen once per chunk, outside the unrolled loops
        // (a branch inside them costs even when it is never taken).
        float dvs[32];
        if (factored) {
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 ie = *reinterpret_cast<const float4 *>(iegv + 32 * hp + 4 * s4);
            dvs[4 * s4 + 0] = fr * ie.x;
            dvs[4 * s4 + 1] = fr * ie.y;
            dvs[4 * s4 + 2] = fr * ie.z;
            dvs[4 * s4 + 3] = fr * ie.w;
          }
        } else {
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 gg = *reinterpret_cast<const float4 *>(gcv + 32 * hp + 4 * s4);
            dvs[4 * s4 + 0] = br * __expf(gr - gg.x);
            dvs[4 * s4 + 1] = br * __expf(gr - gg.y);
            dvs[4 * s4 + 2] = br * __expf(gr - gg.z);
            dvs[4 * s4 + 3] = br * __expf(gr - gg.w);
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = (e < lim) ? x[e] * dvs[e] : 0.f;
        if (rl < 64) {
          float4 *dst = reinterpret_cast<float4 *>(AF + r * LDA + 32 * hp);
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4)
            dst[s4] = make_float4(x[4 * s4], x[4 * s4 + 1], x[4 * s4 + 2], x[4 * s4 + 3]);
        } else {
          st_row32_sw128(sm + Lay::P + s * kTileBytes, r, hp, x);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[B_D1E]);
      group_bar(kBar);
      // ---- Y = (I + A)^{-1}
      invert_unit_lower(AF, reinterpret_cast<float *>(sm + Lay::SCR), pt, kBar);
#ifdef GDR_TC_DEBUG
      for (int hp = hp0; hp < 2; hp += kHalfStep)
        if (rl < 64) DBG_ROW(12288 + 32 * hp, 64, AF + rl * LDA + 32 * hp);
#endif
      // ---- T (lanes 0-63) and T' (lanes 64-127) as bf16 operands
      for (int hp = hp0; hp < 2; hp += kHalfStep) {
        const int r = rl & 63;
        uint8_t *tile = sm + (rl < 64 ? Lay::T : Lay::TP);
        float x[32];
        const float4 *yr = reinterpret_cast<const float4 *>(AF + r * LDA + 32 * hp);
        const float4 *b4 = reinterpret_cast<const float4 *>(bs + 32 * hp);
        const float4 *e4 = reinterpret_cast<const float4 *>(egv + 32 * hp);
        if (rl < 64) {
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 y = yr[s4], bb = b4[s4];
            x[4 * s4 + 0] = y.x * bb.x;
            x[4 * s4 + 1] = y.y * bb.y;
            x[4 * s4 + 2] = y.z * bb.z;
            x[4 * s4 + 3] = y.w * bb.w;
          }
        } else {
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 y = yr[s4], bb = b4[s4], ee = e4[s4];
            x[4 * s4 + 0] = y.x * (bb.x * ee.x);
            x[4 * s4 + 1] = y.y * (bb.y * ee.y);
            x[4 * s4 + 2] = y.z * (bb.z * ee.z);
            x[4 * s4 + 3] = y.w * (bb.w * ee.w);
          }
        }
        st_row32_sw128(tile, r, hp, x);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_TRDY]);
      group_bar(kBar);
      if (pt == 0) mbar_arrive(&bars[B_EMPTY + s]);  // g, beta of this stage no longer read
      // ---- -W^T -> bf16 MN-major operand (row j = this thread's lane)
      if (!group_wait(kBar, &bars[B_WTF], ph, abort_flag, lane)) break;
      tc_fence_after();
      for (int hp = hp0; hp < 2; hp += kHalfStep) {
        float x[32];
        tmem_ld32(lane_base + TM_WT + 32 * hp, x);
        DBG_ROW(16384 + 32 * hp, 64, x);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = -x[e];
        st_row32_sw128(sm + Lay::WT, rl, hp, x);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_WTB]);
    }
  } else if (warp < 4) {
    // ================================================================ state group
    const int i = tid;  // TMEM lane = value channel
    const int lrow = i;
    (void)lrow;
    constexpr uint32_t kBar = 2;
    bool ok = true;
    // Gate factors of chunk c for this group: e^{gc_r} and e^{gc_last - gc_r}
    // into SVEC[c & 1], and the chunk's total decay e^{gc_last}.  Computed
    // from the staged g with the prep group's scan (bit-identical values);
    // the stage's TMA barrier cannot run ahead of this group.
    auto chunk_vectors = [&](int c, float &dl) -> bool {
      if (!group_wait(kBar, &bars[B_FULL + (c & 1)], (c >> 1) & 1, abort_flag, lane))
        return false;
      float *sv = reinterpret_cast<float *>(sm + Lay::SVEC + (c & 1) * 512);
      if (warp == 0) {
        const float *gs = reinterpret_cast<const float *>(sm + Lay::GS + (c & 1) * 512);
        float x0, x1;
        const float gl = chunk_cumsum(gs, lane, x0, x1);
        sv[lane] = __expf(x0);
        sv[lane + 32] = __expf(x1);
        sv[64 + lane] = __expf(gl - x0);
        sv[64 + lane + 32] = __expf(gl - x1);
      }
      group_bar(kBar);
      dl = sv[63];
      return true;
    };
    // S_b = bf16(S) for the next chunk's MMAs, and S <- S * dl (that chunk's
    // decay, applied before its state update accumulates onto S).  The
    // source (S0 in global memory, or S in TMEM) is chosen outside the
    // unrolled loops.
    auto state_cols = [&](int q, const float (&x)[32], float dl) {
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
    };
    auto state_pass = [&](const float *src_global, float dl) {
      if (src_global) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[32];
          const float4 *s4 = reinterpret_cast<const float4 *>(src_global + 32 * q);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 v = s4[e];
            x[4 * e] = v.x;
            x[4 * e + 1] = v.y;
            x[4 * e + 2] = v.z;
            x[4 * e + 3] = v.w;
          }
          state_cols(q, x, dl);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          state_cols(q, x, dl);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[B_SBR]);
    };
    {
      float dl;
      if (!chunk_vectors(0, dl)) {
        ok = false;
      } else if (a.S0) {
        state_pass(a.S0 + ((size_t)bh * DV + i) * DK, dl);
      } else {
        // zero initial state: write zeros through the same path
        float z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0.f;
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = 0u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tmem_st16u(lane_base + TM_SB + 16 * q, u);
          tmem_st16(lane_base + TM_S + 32 * q, *reinterpret_cast<float(*)[16]>(z));
          tmem_st16(lane_base + TM_S + 32 * q + 16, *reinterpret_cast<float(*)[16]>(z + 16));
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[B_SBR]);
      }
    }
    for (int c = 0; ok && c < n; ++c) {
      const uint32_t ph = c & 1;
      const float *sv = reinterpret_cast<const float *>(sm + Lay::SVEC + (c & 1) * 512);
      const float *egv = sv, *eglv = sv + 64;
      // ---- V'^T -> bf16 operands (plain and decayed to the chunk end)
      if (!group_wait(kBar, &bars[B_VPF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      {
        float x[64];
        tmem_ld64(lane_base + TM_UV, x);
        DBG_ROW(40960, 64, x);
        DBG_ROW(40960 + 32, 64, x + 32);
        st_row32_sw128(sm + Lay::VP, i, 0, x);
        st_row32_sw128(sm + Lay::VP, i, 1, x + 32);
        const float4 *e4 = reinterpret_cast<const float4 *>(eglv);
#pragma unroll
        for (int s4 = 0; s4 < 16; ++s4) {
          const float4 e = e4[s4];
          x[4 * s4] *= e.x;
          x[4 * s4 + 1] *= e.y;
          x[4 * s4 + 2] *= e.z;
          x[4 * s4 + 3] *= e.w;
        }
        st_row32_sw128(sm + Lay::VPD, i, 0, x);
        st_row32_sw128(sm + Lay::VPD, i, 1, x + 32);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_VPR]);
      // ---- updated S -> S_b and the next chunk's decay, or the final state
      if (!group_wait(kBar, &bars[B_SF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      if (c + 1 < n) {
        float dl;
        if (!chunk_vectors(c + 1, dl)) { ok = false; break; }
#ifdef GDR_TC_DEBUG
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          DBG_ROW(57344 + 32 * q, 128, x);
        }
#endif
        state_pass(nullptr, dl);
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
      // ---- O = O_a Diag(e^{gc}) + O_b -> bf16, stored straight to o: lanes
      //      i, i^1 swap values so each lane writes two adjacent channels of
      //      one token (a warp writes 2 tokens x 64 contiguous bytes)
      if (!group_wait(kBar, &bars[B_OF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      {
        const int t0 = c * C;
        const size_t tok0 = ((size_t)b * T + t0) * H + h;
        uint32_t *o32 = reinterpret_cast<uint32_t *>(a.o);
        const int chpair = i & ~1;
        const bool full = t0 + C <= T;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float xa[32], xb[32];
          {
            float a0[16], a1[16], b0[16], b1[16];
            tmem_ld16(lane_base + TM_OA + 32 * q, a0);
            tmem_ld16(lane_base + TM_OA + 32 * q + 16, a1);
            tmem_ld16(lane_base + TM_O + 32 * q, b0);
            tmem_ld16(lane_base + TM_O + 32 * q + 16, b1);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              xa[e] = a0[e];
              xa[16 + e] = a1[e];
              xb[e] = b0[e];
              xb[16 + e] = b1[e];
            }
          }
          const float4 *e4 = reinterpret_cast<const float4 *>(egv + 32 * q);
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 ev = e4[s4];
            xa[4 * s4 + 0] = ev.x * xa[4 * s4 + 0] + xb[4 * s4 + 0];
            xa[4 * s4 + 1] = ev.y * xa[4 * s4 + 1] + xb[4 * s4 + 1];
            xa[4 * s4 + 2] = ev.z * xa[4 * s4 + 2] + xb[4 * s4 + 2];
            xa[4 * s4 + 3] = ev.w * xa[4 * s4 + 3] + xb[4 * s4 + 3];
          }
          DBG_ROW(49152 + 32 * q, 64, xa);
          // full chunks store unconditionally; only a ragged last chunk
          // takes the guarded loop (chosen outside the unrolled loops)
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float lo = xa[2 * e], hi = xa[2 * e + 1];  // tokens 32q+2e, +1
            const float send = (i & 1) ? lo : hi;
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            w[e] = (i & 1) ? pack_bf16(recv, hi) : pack_bf16(lo, recv);
          }
          uint32_t *dst = o32 + (((tok0 + (size_t)(32 * q + (i & 1)) * H) * DV + chpair) >> 1);
          const size_t tstep = (size_t)H * DV;  // 32-bit words between tokens t and t + 2
          if (full) {
#pragma unroll
            for (int e = 0; e < 16; ++e) __stcs(dst + e * tstep, w[e]);
          } else {
            const int rem = T - t0 - 32 * q - (i & 1);  // tokens left for this lane's parity
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (2 * e < rem) __stcs(dst + e * tstep, w[e]);
          }
        }
      }
      tc_fence_before();
    }
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

// 4-D map over a [B, T, H, d] bf16 tensor, box = 64 tokens x 64 channels,
// 128-byte swizzle (the layout the MMA descriptors expect).
bool make_map(CUtensorMap *m, const void *base, int B, int T, int H, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B,
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
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.B, a.T, a.H, DK) || !make_map(&mk, a.k, a.B, a.T, a.H, DK) ||
      !make_map(&mv, a.v, a.B, a.T, a.H, DV))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gdr_chunk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  gdr_chunk_tc_kernel<<<(unsigned)((size_t)a.B * a.H), kThreads, kSmemBytes, stream>>>(mq, mk, mv,
                                                                                       a);
  return cudaGetLastError();
}

}  // namespace gdr

#ifdef GDR_TC_DEBUG
extern "C" int gdr_debug_set_buffer(float *p, int chunk) {
  if (cudaMemcpyToSymbol(gdr::g_dbg, &p, sizeof p) != cudaSuccess) return 1;
  return cudaMemcpyToSymbol(gdr::g_dbg_chunk, &chunk, sizeof chunk) != cudaSuccess;
}
#endif
