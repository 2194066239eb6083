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
//   P    = tril_incl(D1_QK[r][s] e^{gc_r - gc_s})        -> bf16, smem
//   Y    = (I + A)^{-1}  (16x16 diagonal blocks by forward substitution,
//                          off-diagonal blocks with mma.sync TF32)
//   T    = Y Diag(beta),  T' = T Diag(e^{gc})             -> bf16, smem
//          (scalar gates: T' also carries the scale sigma of S_b, below)
//   Z    = S_b K^T                          (tcgen05, A = S_b from TMEM)
//   V'^T = V^T T^T - Z T'^T                 (= U^T - S_b W^T with W = T' K)
//          (scalar gates: T' is stored negated and Z enters as it is)
//   O^T  = (S_b Q^T) Diag(e^{gc}) + V'^T P^T
//   S    = e^{gc_last} S + (V'^T Diag(e^{gc_last - gc})) K   (fp32 TMEM acc)
//
// W is never formed: S_b W^T = (S_b K^T) T'^T moves that product onto the
// state side, where it costs one small MMA and one TMEM conversion.  S_b is
// the bf16 copy of the fp32 state, kept in TMEM as the A operand; V'^T's two
// bf16 copies (plain, and decayed to the chunk end) are written back into
// TMEM as well, so every MMA of the state side takes A from TMEM.  Measured
// on the B200: consecutive k-steps into one accumulator wait on each other
// (about 73 cycles each with A in TMEM, 165 with A in shared memory, for
// N = 64 as for N = 128), while independent accumulators overlap; Z and O_a
// are therefore issued with their k-steps interleaved.
//
// The fp32 state is held as S = sigma * S_tmem.  A chunk's decay only
// changes sigma (and scales the next update by 1 / sigma), so S_tmem is
// rewritten only when sigma falls below 2^-40, where the decay is folded
// back into it.  The bf16 copy is S_b = bf16(S_tmem); sigma enters through
// T' and the O epilogue's e^{gc}, which the K/Q producer writes as
// sigma e^{gc} from the same scale sequence (replayed in the same fp32
// operations from the chunk decays).
//
// Warp roles (one CTA per (b, h), 384 threads):
//   warps 0-3  "state" group (TMEM lanes = value channels): Z -> bf16 in
//              TMEM, O_a scaled in place (O_b then accumulates onto it),
//              V'^T -> bf16 operands in TMEM, S -> S_b, O epilogue (each
//              warp stages its 32 channels and stores them with one TMA
//              store); O, T, T' and P have two buffers, so that neither the
//              epilogue of a chunk nor the prep group's next T waits on the
//              state side's progress;
//   warps 4-7  "prep" group, one chunk ahead: gate cumsum, A/P epilogue,
//              (I + A)^{-1} with T/T' written straight from it;
//   warp 8     TMA producer of the K/Q stages (three) + g/beta loads;
//   warp 9     state-side MMA issuer (Z with O_a, U^T = V^T T^T, V'^T, S,
//              O_b; one thread);
//   warp 10    TMA producer of V (one stage);
//   warp 11    prep-side MMA issuer (D1, one thread): an issue can stall
//              while the tensor core's queue is full, which must not hold up
//              the prep group.
// No TMA load uses cluster multicast.  Hand-offs are mbarriers; every wait
// is bounded (time-out -> device status word, abort flag, orderly unwind,
// TMEM freed).
#include <cudaTypedefs.h>

#include <mutex>

#include "gdr_internal.cuh"
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using namespace sm100;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kVWarp = 10, kPrepMmaWarp = 11;
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s per wait
constexpr uint32_t kTileBytes = 64 * 128;     // one 64 x 64 bf16 tile
constexpr uint32_t kKQTx = 4 * kTileBytes, kVTx = 2 * kTileBytes;
constexpr float kSafeDecay = 80.f;            // e^{80} is finite in fp32
constexpr float kScaleFloor = 0x1p-40f;       // smallest state scale sigma kept
// Row stride (floats) of the fp32 A matrix: rows stay 16-byte aligned and
// 16 consecutive rows hit distinct 16-byte bank groups pairwise.
constexpr int LDA = 68;

// Gate vectors of a stage, written by the K/Q producer (float offsets):
// gc = cumulative log decay from the chunk start, e^{gc}, e^{-gc},
// e^{gc_last - gc}, beta.  Per-channel gates (PC) use gc = 0 and factors 1
// here (the decay is inside the scaled K/Q tiles) and add, per key channel,
// e^{m} and e^{gc_last - m} (m = the cumulative decay at row 31).
constexpr int kGateGc = 0, kGateEg = 64, kGateIeg = 128, kGateEgl = 192, kGateBeta = 256,
              kGateEm = 320, kGateEgm = 448;
// Scalar gates only (PC keeps e^{m} there): sigma_c e^{gc}, where sigma_c is
// the scale of the bf16 state copy S_b the chunk's MMAs read (the state
// group forms S_b from S_tmem unscaled; T' and the O epilogue carry sigma).
constexpr int kGateSEg = 320;
// Prologue instance only (scalar gates): the tiles hold raw K, Q, and each
// token's 1 / |k| and 1 / |q| (rk, rq) ride on the per-token vectors instead:
// once a stage has landed, Ieg and Egl are multiplied by rk in place
// (columns of A and P, the state update's rows), T' takes sigma e^{gc} rk
// (SEgK), the O epilogue sigma e^{gc} rq (SEgQ), and the A / P rows take
// rk / rq from their own vectors.
constexpr int kGateRk = 384, kGateRq = 448, kGateSEgQ = 512, kGateSEgK = 576;
// The state group's copy per chunk (float offsets): e^{gc}, e^{gc_last - gc};
// PC adds e^{m} and e^{gc_last - m}.
constexpr int kSvEg = 0, kSvEgl = 64, kSvEm = 128, kSvEgm = 256;

// Per-variant configuration: K/Q stages and the shared-memory layout (byte
// offsets from a 1024-byte aligned base).  PC (per-channel gates) holds, per
// stage, the scaled K~, Q~ tiles in place of K, Q and K^ in its own tiles,
// each scaling warp's fp32 gate rows (its 64 channels, rows 0-31 and 32-63
// of the chunk being scaled, each half refilled with the next chunk's as
// soon as it has been read), and shares T with T' (identical without a
// scalar decay).  V'^T never goes to shared memory: its bf16 operand copies
// are written back into TMEM (the MMAs that read it take A from TMEM).
template <bool PC>
struct Cfg {
  static constexpr int kStages = PC ? 2 : 3;
  static constexpr uint32_t kGateBytes = (PC ? 576 : 640) * 4;
  static constexpr uint32_t kSvecBytes = (PC ? 512 : 128) * 4;
  static constexpr uint32_t KQ = 0;                                          // [K_h0|Q_h0|K_h1|Q_h1]
  static constexpr uint32_t KH = KQ + kStages * 4 * kTileBytes;              // PC: [Kh_h0|Kh_h1]
  static constexpr uint32_t GT = KH + (PC ? kStages * 2 * kTileBytes : 0);   // PC: g [2][2][32][64]
  static constexpr uint32_t V = GT + (PC ? 64 * 128 * 4 : 0);                // [V_h0|V_h1]
  static constexpr uint32_t T = V + 2 * kTileBytes;                          // T  K-major [r][s], x2
  static constexpr uint32_t TP = T + (PC ? 0 : 2 * kTileBytes);              // T' K-major, x2
  static constexpr uint32_t P = TP + 2 * kTileBytes;                         // P  K-major, x2
  static constexpr uint32_t STG = P + 2 * kTileBytes;                        // o staging (4 x 4 KB)
  static constexpr uint32_t AF = STG + 2 * kTileBytes;                       // fp32 A, D blocks
  static constexpr uint32_t SCR = AF + 64 * LDA * 4;                         // inverse scratch
  static constexpr uint32_t GS = SCR + (512 + 4 * 256) * 4;                  // gate vectors
  static constexpr uint32_t SVEC = GS + kStages * kGateBytes;                // x3 (state group)
  static constexpr uint32_t BAR = SVEC + 3 * kSvecBytes;                     // mbarriers
  static constexpr uint32_t MISC = BAR + 40 * 8;                             // tmem base, abort
  static constexpr uint32_t END = MISC + 16;
  static constexpr size_t kSmemBytes = END + 1024;
  static_assert(V % 1024 == 0 && T % 1024 == 0 && STG % 1024 == 0 && AF % 1024 == 0 &&
                    GT % 1024 == 0,
                "tile alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// mbarrier slots
enum {
  B_FULL = 0,          // [3] K/Q + g/beta of a stage landed            (1 + tx)
  B_EMPTY = 3,         // [3] K/Q stage free (state MMA commit)         (commit)
  B_VFULL = 6,         // V landed                                      (1 + tx)
  B_VEMPTY,            // V free (commit after U)                       (commit)
  B_D1F,               // D1 written                                    (commit, prep side)
  B_D1E,               // D1 read by the prep group                     (4 warps)
  B_TRDY,              // [2] T, T' and P of a chunk written (buffer c % 2) (4 warps)
  B_UF = B_TRDY + 2,   // [2] U^T written (T buffer c % 2 read)         (commit)
  B_ZF = B_UF + 2,     // Z and O_a written                             (commit)
  B_ZR,                // Z (or -Z) bf16 operand in TMEM                (4 warps)
  B_VPF,               // V'^T complete                                 (commit)
  B_VPR,               // V'^T bf16 operands (and O_a scaled) in TMEM   (4 warps)
  B_SF,                // state update complete                         (commit)
  B_OF,                // O (O_a scaled + O_b) complete                 (commit)
  B_SBR,               // S_b in TMEM for the next chunk                (4 warps)
  B_OE,                // [2] O buffer c % 2 read by the epilogue       (4 warps)
  B_PE = B_OE + 2,     // [2] P buffer free (after O_b)                 (commit)
  B_TPE = B_PE + 2,    // [2] T' buffer free (after V')                 (commit)
  B_FIN = B_TPE + 2,   // final drain, state-side issuer                (commit)
  B_FIN2,              // final drain, prep-side issuer                 (commit)
  B_SCALED,            // [2] PC: scaled K~, Q~, K^ of a stage written  (2 warps)
  B_GF = B_SCALED + 2, // [4] PC: gate rows of a scaling warp landed    (1 + tx)
                       //     (warp w, rows 0-31 / 32-63: 2 w + half)
  B_NORM = B_GF,       // [3] prologue (scalar gates): token norms of a
                       //     stage folded into its vectors (prep group, 1 thread)
  B_COUNT = B_GF + 4
};
static_assert(B_COUNT <= 40, "barrier slots");

// TMEM column map (512 allocated; 1 CTA per SM).  UV holds U^T, then V'^T
// in fp32, then its two bf16 operand copies (plain in columns 0-31, decayed
// in 32-63), converted in place.  O has two buffers (chunk c in c % 2):
// O_a = S_b Q^T, scaled in place by the state group, then O_b accumulated
// onto it, so the epilogue of chunk c never holds up chunk c + 1.
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_Z = 192, TM_O0 = 256, TM_UV = 320, TM_O1 = 384,
                   TM_D1 = 448;

constexpr uint32_t ID_D1 = idesc_bf16(128, 64, 0, 0);
constexpr uint32_t ID_U = idesc_bf16(128, 64, 1, 0);
constexpr uint32_t ID_N64 = idesc_bf16(128, 64, 0, 0);
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

// 16 TMEM lanes x 32 columns (shape 16x256b, 4 repeats): for column group
// k (8 columns), thread t holds lane t / 4 at columns 8 k + 2 (t % 4) and
// + 1 (v[4 k], v[4 k + 1]) and lane t / 4 + 8 at the same columns
// (v[4 k + 2], v[4 k + 3]).  No wait.
__device__ __forceinline__ void tmem_ld16x256b_x4(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Four 8x8 b16 matrices stored transposed: register j of thread t holds
// elements (t / 4, 2 (t % 4)) and (t / 4, 2 (t % 4) + 1) of matrix j, which
// land in memory rows 2 (t % 4) and 2 (t % 4) + 1, column t / 4; threads
// 8 j .. 8 j + 7 give the 16-byte aligned row addresses of matrix j.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t r0, uint32_t r1,
                                                  uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr),
               "r"(r0), "r"(r1), "r"(r2), "r"(r3)
               : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t *v) {
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

// Barrier over the prep warpgroup (id 3, 128 threads) that also ORs a
// failure flag, so that the group leaves its loop together (a warp left
// behind at a named barrier would never return).
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


// Bounded wait that also gives up as soon as another role has aborted.
// The thread blocks inside try_wait (for the hardware's default time)
// between checks; a long suspend hint was measured to wake it later after
// the phase completes.  The slow path is out of line: it would otherwise be
// copied into every wait site of the hot loops.
__device__ __noinline__ bool wait_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
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

// End-of-kernel drains (bounded, cold): out of line as well.
__device__ __noinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  return mbar_wait_bounded(bar, parity, kWaitNs);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag);
}

// Waits for N phases at once.  The non-blocking probes are independent, so
// their latencies overlap (a chain of single waits costs each probe's full
// latency in turn); only when one of them is incomplete does the thread take
// the bounded, abort-aware path barrier by barrier.  Uniform per warp when
// every lane calls it.  A parity of 1 on a barrier that has not completed
// its first phase passes at once: the first chunks' "previous phase" waits
// rely on that.
template <int N>
__device__ __forceinline__ bool wait_all(uint64_t *const (&bar)[N], const uint32_t (&parity)[N],
                                         volatile int *abort_flag) {
  bool done = true;
#pragma unroll
  for (int j = 0; j < N; ++j) done &= mbar_test_wait(bar[j], parity[j]);
  if (done) return true;
#pragma unroll
  for (int j = 0; j < N; ++j)
    if (!wait_or_abort(bar[j], parity[j], abort_flag)) return false;
  return true;
}

// Warp-wide wait for one phase (false on time-out or once an abort was
// raised anywhere in the CTA while waiting).  Every lane polls the same
// barrier, so the result is warp-uniform without a shuffle (chained shuffles
// were measured at several hundred cycles each in this kernel).  Warps wait
// on their own: a group barrier after every wait would make each warp wait
// for the slowest one as well.  A phase that is already complete returns at
// once without reading the abort flag (that read, on every hand-off, cost
// about 4 % of the kernel): a role that keeps finding its phases complete
// goes on, and the first wait that has to sleep sees the flag.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity,
                                          volatile int *abort_flag, int lane) {
  (void)lane;
  return wait_or_abort(bar, parity, abort_flag);
}

// One arrival per warp: every lane's earlier writes and fences are ordered
// before lane 0's (release) arrive by the warp barrier.  Per-thread
// arrivals on one barrier word serialise: a group of 128 was measured at
// several hundred cycles per hand-off.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// One warp: cumulative log decay of a chunk (g[64] -> gc[64] in log space,
// inclusive prefix sum) held as lanes r and r + 32; returns the chunk total.
// Used by the K/Q producer only, which runs chunks ahead of its consumers.
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

// ---------------------------------------------------------------- inverse
// Output of the inverse: T = Y Diag(beta) and T' = T Diag(eg) as bf16
// K-major 128B-swizzled tiles [r][s] (eg: e^{gc}, scalar gates sigma e^{gc}).
struct TOut {
  uint8_t *t, *tp;
  const float *beta, *eg;  // [64]
};

// The tensor core reads the top 19 bits of a tf32 operand register, i.e.
// fp32 truncated toward zero (error below 2^-10 relative, under the bf16
// rounding T and T' get afterwards), so no conversion instruction is spent.
__device__ __forceinline__ uint32_t to_tf32(float x) { return __float_as_uint(x); }

// D += A(16x8, row) * B(8x8, col), tf32 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// mma.sync m16n8k8 TF32 fragments of one warp (g = lane / 4, tq = lane % 4).
// The k index is permuted identically in A and B (fragment slot tq holds
// k = 2 tq, slot tq + 4 holds k = 2 tq + 1), which leaves the product
// unchanged and makes each lane's two A elements of a row adjacent.
struct Frag {
  int g, tq;
  float *scr;  // warp-private 2 x [16][8] fp32 scratch
  // A fragment of the 16x8 block at (row0, col0) of a row-major matrix.
  __device__ __forceinline__ void a(const float *M, int ld, int row0, int col0,
                                    uint32_t (&af)[4]) const {
    const float2 lo = *reinterpret_cast<const float2 *>(M + (row0 + g) * ld + col0 + 2 * tq);
    const float2 hi = *reinterpret_cast<const float2 *>(M + (row0 + g + 8) * ld + col0 + 2 * tq);
    af[0] = to_tf32(lo.x);
    af[1] = to_tf32(hi.x);
    af[2] = to_tf32(lo.y);
    af[3] = to_tf32(hi.y);
  }
  // B fragments (two k-steps) of a 16x8 block of a row-major matrix.
  __device__ __forceinline__ void b(const float *blk, int ld, uint32_t (&bf)[2][2]) const {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      bf[ks][0] = to_tf32(blk[(8 * ks + 2 * tq) * ld + g]);
      bf[ks][1] = to_tf32(blk[(8 * ks + 2 * tq + 1) * ld + g]);
    }
  }
  // 16x8 accumulator fragments -> B fragments, through the scratch (one
  // shared-memory round trip, for one or two fragments).
  __device__ __forceinline__ void put(float *m, const float (&cf)[4]) const {
    m[g * 8 + 2 * tq] = cf[0];
    m[g * 8 + 2 * tq + 1] = cf[1];
    m[(g + 8) * 8 + 2 * tq] = cf[2];
    m[(g + 8) * 8 + 2 * tq + 1] = cf[3];
  }
  __device__ __forceinline__ void to_b(const float (&c0)[4], uint32_t (&b0)[2][2]) const {
    put(scr, c0);
    __syncwarp();
    b(scr, 8, b0);
    __syncwarp();
  }
  __device__ __forceinline__ void to_b2(const float (&c0)[4], const float (&c1)[4],
                                        uint32_t (&b0)[2][2], uint32_t (&b1)[2][2]) const {
    put(scr, c0);
    put(scr + 128, c1);
    __syncwarp();
    b(scr, 8, b0);
    b(scr + 128, 8, b1);
    __syncwarp();
  }
};

// acc (+)= A (16 x 16 block at (row0, col0), two k-steps) * B (16 x 8), with
// one accumulator per k-step (the caller sums them).
__device__ __forceinline__ void mma_blk(const Frag &f, const float *M, int ld, int row0, int col0,
                                        const uint32_t (&bf)[2][2], float (&acc0)[4],
                                        float (&acc1)[4]) {
  uint32_t a0[4], a1[4];
  f.a(M, ld, row0, col0, a0);
  f.a(M, ld, row0, col0 + 8, a1);
  mma_tf32_16x8x8(acc0, a0, bf[0]);
  mma_tf32_16x8x8(acc1, a1, bf[1]);
}

// Two adjacent columns s, s + 1 (s even) of row r of T and T' (kNegTp: -T',
// which lets the state side use +Z as its operand).
template <bool kNegTp>
__device__ __forceinline__ void store_t2(const TOut &o, int r, int s, float y0, float y1) {
  const float2 b = *reinterpret_cast<const float2 *>(o.beta + s);
  const float2 e = *reinterpret_cast<const float2 *>(o.eg + s);
  const float t0 = y0 * b.x, t1 = y1 * b.y;
  const uint32_t off = sw128_off(r, s);
  *reinterpret_cast<uint32_t *>(o.t + off) = pack_bf16(t0, t1);
  const float ex = kNegTp ? -e.x : e.x, ey = kNegTp ? -e.y : e.y;
  *reinterpret_cast<uint32_t *>(o.tp + off) = pack_bf16(t0 * ex, t1 * ey);
}

// (I + A)^{-1} for the strictly lower 64x64 fp32 A in AF (row stride LDA,
// zero above the diagonal) with the 4-warp prep group (local thread t),
// written as T and T' (their blocks above the block diagonal stay zero from
// the kernel's start), in two steps with a group barrier between them:
//  1. D_bb = (I + A_bb)^{-1} by forward substitution, in the two warps
//     that wrote A (two blocks each), stored over A_bb in AF and, scaled,
//     into T and T';
//  2. the off-diagonal blocks in two doubling levels (below), with mma.sync.
//     (An fp32 CUDA-core sweep was faster alone but, competing for issue
//     slots with the state group, slower in the kernel.)
__device__ void invert_diag(float *AF, const TOut &o, int pw, int lane) {
  // warp pw (0 or 1) has just written A rows 32 pw .. 32 pw + 31: lanes
  // 0-15 invert block 2 pw, lanes 16-31 block 2 pw + 1 (lane c % 16 owns
  // column c of its block)
  const int w = 2 * pw + (lane >> 4), c = lane & 15;
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = (i == c) ? 1.f : 0.f;
  const float *Ab = AF + (16 * w) * LDA + 16 * w;
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int k4 = 0; k4 < (i + 3) / 4; ++k4) {
      const float4 av = *reinterpret_cast<const float4 *>(Ab + i * LDA + 4 * k4);
      if (4 * k4 + 0 < i) acc0 += av.x * x[4 * k4 + 0];
      if (4 * k4 + 1 < i) acc1 += av.y * x[4 * k4 + 1];
      if (4 * k4 + 2 < i) acc0 += av.z * x[4 * k4 + 2];
      if (4 * k4 + 3 < i) acc1 += av.w * x[4 * k4 + 3];
    }
    x[i] = (i > c) ? -(acc0 + acc1) : x[i];
  }
  __syncwarp();  // every lane has read its A_ww
  float *Yb = AF + (16 * w) * LDA + 16 * w;
#pragma unroll
  for (int i = 0; i < 16; ++i) Yb[i * LDA + c] = x[i];
  (void)o;  // T and T' of the diagonal blocks: diag_to_t, after the barrier
}

// T and T' of the four diagonal blocks from D_bb in AF, spread over the 128
// prep threads (one row pair of four columns each, paired bf16 stores).
template <bool kNegTp>
__device__ __forceinline__ void diag_to_t(const float *AF, const TOut &o, int t) {
  const int blk = t >> 5, r = (t >> 1) & 15, c0 = 8 * (t & 1);  // 8 columns per thread
  const int row = 16 * blk + r, col = 16 * blk + c0;
  const float *src = AF + row * LDA + col;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 y = *reinterpret_cast<const float2 *>(src + 2 * p);
    store_t2<kNegTp>(o, row, col + 2 * p, y.x, y.y);
  }
}

// Off-diagonal blocks of Y by two doubling levels (with every D_bb in AF):
//  level 1:  Y_10 = -D_11 A_10 D_00,   Y_32 = -D_33 A_32 D_22;
//  level 2:  [Y_20 Y_21; Y_30 Y_31] = -[D_22 0; Y_32 D_33] R,
//            R = [A_20 A_21; A_30 A_31] [D_00 0; Y_10 D_11].
// Each warp takes one 8-column strip per level (mma.sync TF32, fp32
// accumulation); Y_10 and Y_32 reach level 2 through the shared scratch
// `ysc` ([2][16][16]); every block is written, scaled, to T and T'.
template <bool kNegTp>
__device__ void invert_level1(const float *AF, float *ysc, float *scr, const TOut &o, int t) {
  const int warp = t >> 5, lane = t & 31;
  const Frag f{lane >> 2, lane & 3, scr + warp * 256};
  const int jb = warp < 2 ? 0 : 2, blk = jb + 1, cs = 8 * (warp & 1);
  uint32_t bf[2][2], rb[2][2];
  f.b(AF + (16 * jb) * LDA + 16 * jb + cs, LDA, bf);  // D_jj strip
  float r0[4] = {0.f, 0.f, 0.f, 0.f}, r1[4] = {0.f, 0.f, 0.f, 0.f};
  mma_blk(f, AF, LDA, 16 * blk, 16 * jb, bf, r0, r1);  // A_{blk,jb} D_jj
  const float r[4] = {r0[0] + r1[0], r0[1] + r1[1], r0[2] + r1[2], r0[3] + r1[3]};
  f.to_b(r, rb);
  float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
  mma_blk(f, AF, LDA, 16 * blk, 16 * blk, rb, y0, y1);  // D_{blk,blk} R
  const float y[4] = {-(y0[0] + y1[0]), -(y0[1] + y1[1]), -(y0[2] + y1[2]), -(y0[3] + y1[3])};
  float *yo = ysc + (jb >> 1) * 256 + cs;  // [16][16]
  yo[f.g * 16 + 2 * f.tq] = y[0];
  yo[f.g * 16 + 2 * f.tq + 1] = y[1];
  yo[(f.g + 8) * 16 + 2 * f.tq] = y[2];
  yo[(f.g + 8) * 16 + 2 * f.tq + 1] = y[3];
  store_t2<kNegTp>(o, 16 * blk + f.g, 16 * jb + cs + 2 * f.tq, y[0], y[1]);
  store_t2<kNegTp>(o, 16 * blk + f.g + 8, 16 * jb + cs + 2 * f.tq, y[2], y[3]);
}

// Level 2, after a group barrier (Y_10 and Y_32 in ysc): warp w takes the
// columns 8 w .. 8 w + 7 of the lower-left 32x32 block.
template <bool kNegTp>
__device__ void invert_level2(const float *AF, const float *ysc, float *scr, const TOut &o,
                              int t) {
  const int warp = t >> 5, lane = t & 31;
  const Frag f{lane >> 2, lane & 3, scr + warp * 256};
  const int jb = warp >> 1, cs = 8 * (warp & 1), col = 16 * jb + cs;
  float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};  // R_2 (block row 2)
  float q0[4] = {0.f, 0.f, 0.f, 0.f}, q1[4] = {0.f, 0.f, 0.f, 0.f};  // R_3 (block row 3)
  uint32_t bf[2][2];
  if (jb == 0) {  // strip of [D_00; Y_10]
    f.b(AF + cs, LDA, bf);
    mma_blk(f, AF, LDA, 32, 0, bf, p0, p1);
    mma_blk(f, AF, LDA, 48, 0, bf, q0, q1);
    f.b(ysc + cs, 16, bf);
  } else {  // strip of [0; D_11]
    f.b(AF + 16 * LDA + 16 + cs, LDA, bf);
  }
  mma_blk(f, AF, LDA, 32, 16, bf, p0, p1);
  mma_blk(f, AF, LDA, 48, 16, bf, q0, q1);
  const float r2[4] = {p0[0] + p1[0], p0[1] + p1[1], p0[2] + p1[2], p0[3] + p1[3]};
  const float r3[4] = {q0[0] + q1[0], q0[1] + q1[1], q0[2] + q1[2], q0[3] + q1[3]};
  uint32_t b2[2][2], b3[2][2];
  f.to_b2(r2, r3, b2, b3);
  float u0[4] = {0.f, 0.f, 0.f, 0.f}, u1[4] = {0.f, 0.f, 0.f, 0.f};
  float v0[4] = {0.f, 0.f, 0.f, 0.f}, v1[4] = {0.f, 0.f, 0.f, 0.f};
  mma_blk(f, AF, LDA, 32, 32, b2, u0, u1);      // D_22 R_2
  mma_blk(f, ysc + 256, 16, 0, 0, b2, v0, v1);  // Y_32 R_2
  mma_blk(f, AF, LDA, 48, 48, b3, v0, v1);      // + D_33 R_3
  store_t2<kNegTp>(o, 32 + f.g, col + 2 * f.tq, -(u0[0] + u1[0]), -(u0[1] + u1[1]));
  store_t2<kNegTp>(o, 40 + f.g, col + 2 * f.tq, -(u0[2] + u1[2]), -(u0[3] + u1[3]));
  store_t2<kNegTp>(o, 48 + f.g, col + 2 * f.tq, -(v0[0] + v1[0]), -(v0[1] + v1[1]));
  store_t2<kNegTp>(o, 56 + f.g, col + 2 * f.tq, -(v0[2] + v1[2]), -(v0[3] + v1[3]));
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

// Largest log2 factor the per-channel tile scaling applies (2^120, well
// inside bf16's range for unit-norm rows); a chunk whose per-channel decay
// over half a chunk goes beyond it (about e^{-83}) reports kStatusRange.
constexpr float kMaxExp2 = 120.f;

// 2^x with the hardware approximation (ex2.approx, the instruction __expf is
// built on); the per-channel scaling keeps its logs in base 2.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- prologue (raw projections in): "Decoding Hybrid Linear Attention
// Architectures", section 3 item 2 (the erase is a projector along a unit
// key) and section 4 (beta in (0, 1), alpha in (0, 1]):
//   q, k <- x / sqrt(|x|^2 + eps),  beta = sigmoid(b),  g = -s_h softplus(a).
constexpr float kNormEps = 1e-6f;

__device__ __forceinline__ float softplus_f(float x) {
  return fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }

// Token norms (prologue), in the prep group.  |k_s|^2 is the diagonal of
// K K^T, which D1 already holds (rows 0-63); |q_r|^2 is summed from the
// landed Q tiles, two threads per token.
__device__ __forceinline__ float sumsq_bf16x8(uint4 x, float ss) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[u]));
    ss = fmaf(f.x, f.x, ss);
    ss = fmaf(f.y, f.y, ss);
  }
  return ss;
}

// Sum of squares of one 128-byte row of a swizzled 64-channel tile.  The
// sum does not depend on the order of the 16-byte chunks, so the swizzle is
// ignored and lane l starts at chunk l % 8, which puts the 8 lanes of a
// 16-byte access phase on distinct banks.
__device__ __forceinline__ float row_sumsq_half(const uint8_t *row, int lane) {
  float s = 0.f;
#pragma unroll
  for (int p = 0; p < 8; ++p)
    s = sumsq_bf16x8(*reinterpret_cast<const uint4 *>(row + ((p + lane) & 7) * 16), s);
  return s;
}

// x[lane] of a register row, by a select tree on the lane's bits.
__device__ __forceinline__ float pick_lane(const float (&x)[32], int lane) {
  float y[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) y[e] = (lane & 1) ? x[2 * e + 1] : x[2 * e];
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = (lane & 2) ? y[2 * e + 1] : y[2 * e];
#pragma unroll
  for (int e = 0; e < 4; ++e) y[e] = (lane & 4) ? y[2 * e + 1] : y[2 * e];
#pragma unroll
  for (int e = 0; e < 2; ++e) y[e] = (lane & 8) ? y[2 * e + 1] : y[2 * e];
  return (lane & 16) ? y[1] : y[0];
}

// Scalar gates of one stage from the per-token log decays (gl0: token lane,
// gl1: token lane + 32) and betas: the cumulative decay gc, e^{gc}, e^{-gc},
// e^{gc_last - gc}, beta and sigma e^{gc} into gv; sig advances to the
// state scale after the chunk (see the state group), replayed in the same
// fp32 operations.  One warp.
__device__ __forceinline__ void write_scalar_gates(float *gv, float gl0, float gl1, float b0,
                                                   float b1, int lane, int c, float &sig) {
  float *gc = gv + kGateGc;
  gc[lane] = gl0;
  gc[lane + 32] = gl1;
  __syncwarp();
  float x0, x1;
  const float gl = chunk_cumsum(gc, lane, x0, x1);
  __syncwarp();
  gc[lane] = x0;
  gc[lane + 32] = x1;
  gv[kGateEg + lane] = __expf(x0);
  gv[kGateEg + lane + 32] = __expf(x1);
  gv[kGateIeg + lane] = __expf(-x0);
  gv[kGateIeg + lane + 32] = __expf(-x1);
  gv[kGateEgl + lane] = __expf(gl - x0);
  gv[kGateEgl + lane + 32] = __expf(gl - x1);
  gv[kGateBeta + lane] = b0;
  gv[kGateBeta + lane + 32] = b1;
  gv[kGateSEg + lane] = sig * __expf(x0);
  gv[kGateSEg + lane + 32] = sig * __expf(x1);
  // the scale after this chunk: 1 after chunk 0 (its decay goes into
  // S_tmem), else sig * decay unless that falls below the floor
  const float nxt = sig * __expf(gl);  // the decay e^{gc_last} as stored above
  sig = (c == 0 || !(nxt >= kScaleFloor)) ? 1.f : nxt;
}

// Per-channel gates, one warp, channels j0 .. j0 + 63 of a chunk (lane l:
// the adjacent pair j0 + 2 l, j0 + 2 l + 1).  g0 / g1: the warp's gate rows
// 0-31 / 32-63 of the chunk ([32][64] fp32 log decay; rows from nv on read as
// zero: past the end of the sequence), landed
// on gf[0] / gf[1] (phase parity ph).  The cumulative log decay gc (log2
// units) of rows 0-31 is formed in place; the reference m = gc at row 31,
// e^{m} and e^{gc_last - m} go into the stage's gate vectors, and the
// operand tiles are scaled in place:
//   K~ = K e^{gc - m},  Q~ = Q e^{gc - m},  K^ = K e^{m - gc}  (bf16),
// so that K~ K^T, Q~ K^T carry e^{gc_r - gc_s} per channel, and with the
// state kept as S Diag(e^{m}), Z and O_a carry e^{gc} (decay from the chunk
// start) and the update V'^T K^ carries e^{m - gc}.  The factors stay within
// e^{|gc_last| / 2}.  Each half is refilled with rows of the chunk at token
// t0n of tensor row bt (none if t0n < 0) as soon as the warp has read it, so
// the load runs
// under the other half's work.  Returns 2 when done, 1 if the wait for rows
// 32-63 gave up (rows 0-31 already refilled), 0 if the first wait gave up.
__device__ __forceinline__ void scale_row(uint8_t *kt, uint8_t *qt, uint8_t *ht, int t, int jc,
                                          float dx, float dy) {
  const float ux = ex2(dx), uy = ex2(dy), vx = ex2(-dx), vy = ex2(-dy);
  const uint32_t off = sw128_off(t, jc);
  uint32_t *kp = reinterpret_cast<uint32_t *>(kt + off);
  uint32_t *qp = reinterpret_cast<uint32_t *>(qt + off);
  const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(kp));
  const float2 qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(qp));
  *kp = pack_bf16(kv.x * ux, kv.y * uy);
  *qp = pack_bf16(qv.x * ux, qv.y * uy);
  *reinterpret_cast<uint32_t *>(ht + off) = pack_bf16(kv.x * vx, kv.y * vy);
}

// Zero the low (lo) and / or high (hi) bf16 of a pair in a tile.
__device__ __forceinline__ void clear_pair(uint8_t *tile, uint32_t off, bool lo, bool hi) {
  uint32_t *p = reinterpret_cast<uint32_t *>(tile + off);
  *p &= (lo ? 0xffff0000u : 0xffffffffu) & (hi ? 0x0000ffffu : 0xffffffffu);
}

// Cold: a channel whose log2 decay factor exceeds kMaxExp2 within the chunk
// (a per-channel decay stronger than the tile scaling can represent).  The
// entries whose factor overflowed are set to zero, so that nothing infinite
// reaches the tensor core; the chunk's results are then not the
// recurrence's, which the range status bit reports.  First half (rows 0-31,
// g0 = cumulative log2 decay): K~ and Q~ carry 2^{gc - m} >= 1.
__device__ __noinline__ void clear_first_half(uint8_t *kt, uint8_t *qt, const float *g0, int jl,
                                              int jc, float mx, float my) {
  for (int t = 0; t < 32; ++t) {
    const float2 gl = *reinterpret_cast<const float2 *>(g0 + t * 64 + jl);
    const bool lo = gl.x - mx > kMaxExp2, hi = gl.y - my > kMaxExp2;
    if (lo || hi) {
      clear_pair(kt, sw128_off(t, jc), lo, hi);
      clear_pair(qt, sw128_off(t, jc), lo, hi);
    }
  }
}

// Second half (rows 32-63, g1 = per-token log decay): K^ carries
// 2^{m - gc} >= 1.
__device__ __noinline__ void clear_second_half(uint8_t *ht, const float *g1, int jl, int jc,
                                               int nv, float mx, float my) {
  constexpr float kLog2e = 1.4426950408889634f;
  float ax = mx, ay = my;
  for (int t = 32; t < 64; ++t) {
    const float2 x = t < nv ? *reinterpret_cast<const float2 *>(g1 + (t - 32) * 64 + jl)
                            : make_float2(0.f, 0.f);
    ax += x.x * kLog2e;
    ay += x.y * kLog2e;
    const bool lo = mx - ax > kMaxExp2, hi = my - ay > kMaxExp2;
    if (lo || hi) clear_pair(ht, sw128_off(t, jc), lo, hi);
  }
}

__device__ int scale_channels(uint8_t *kq, uint8_t *kh, float *g0, float *g1, uint64_t *gf,
                              uint32_t ph, const CUtensorMap *tmG, int h, int bt, int t0n,
                              int nv, float *gv, int j0, int lane, volatile int *abort_flag,
                              unsigned int *status) {
  constexpr float kLog2e = 1.4426950408889634f;
  const int jl = 2 * lane, j = j0 + jl, hh = j >> 6, jc = j & 63;
  uint8_t *kt = kq + (2 * hh) * kTileBytes, *qt = kt + kTileBytes, *ht = kh + hh * kTileBytes;
  if (!warp_wait(&gf[0], ph, abort_flag, lane)) return 0;
  float2 acc = make_float2(0.f, 0.f), first = acc;
#pragma unroll 8
  for (int t = 0; t < 32; ++t) {
    float2 *p = reinterpret_cast<float2 *>(g0 + t * 64 + jl);
    const float2 x = t < nv ? *p : make_float2(0.f, 0.f);
    acc.x += x.x * kLog2e;
    acc.y += x.y * kLog2e;
    *p = acc;
    if (t == 0) first = acc;
  }
  const float2 m = acc;
  gv[kGateEm + j] = ex2(m.x);
  gv[kGateEm + j + 1] = ex2(m.y);
#pragma unroll 4
  for (int t = 0; t < 32; ++t) {
    const float2 gl = *reinterpret_cast<const float2 *>(g0 + t * 64 + jl);
    scale_row(kt, qt, ht, t, jc, gl.x - m.x, gl.y - m.y);
  }
  // the largest factor of rows 0-31 is 2^{gc_0 - m}
  bool out_of_range = false;
  if (__any_sync(0xffffffffu, fmaxf(first.x - m.x, first.y - m.y) > kMaxExp2)) {
    clear_first_half(kt, qt, g0, jl, jc, m.x, m.y);
    out_of_range = true;
  }
  // rows 0-31 read (and written, by the generic proxy): refill
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && t0n >= 0) {
    mbar_arrive_expect_tx(&gf[0], 32 * 64 * 4);
    tma_load_4d(g0, tmG, &gf[0], j0, h, t0n, bt);
  }
  if (!warp_wait(&gf[1], ph, abort_flag, lane)) return 1;
#pragma unroll 4
  for (int t = 32; t < 64; ++t) {
    const float2 x = t < nv ? *reinterpret_cast<const float2 *>(g1 + (t - 32) * 64 + jl)
                            : make_float2(0.f, 0.f);
    acc.x += x.x * kLog2e;
    acc.y += x.y * kLog2e;
    scale_row(kt, qt, ht, t, jc, acc.x - m.x, acc.y - m.y);
  }
  // the largest factor of rows 32-63 is 2^{m - gc_63}
  if (__any_sync(0xffffffffu, fmaxf(m.x - acc.x, m.y - acc.y) > kMaxExp2)) {
    clear_second_half(ht, g1, jl, jc, nv, m.x, m.y);
    out_of_range = true;
  }
  if (out_of_range && lane == 0) atomicOr(status, kStatusRange);
  __syncwarp();
  if (lane == 0 && t0n >= 0) {
    mbar_arrive_expect_tx(&gf[1], 32 * 64 * 4);
    tma_load_4d(g1, tmG, &gf[1], j0, h, t0n + 32, bt);
  }
  gv[kGateEgm + j] = ex2(acc.x - m.x);
  gv[kGateEgm + j + 1] = ex2(acc.y - m.y);
  return 2;
}

// Each SM sub-partition holds a quarter of the register file and three of
// the block's twelve warps: the launch bound caps registers at 168.
template <bool PC, bool ADD, bool PRO, bool STASH>
__global__ void __launch_bounds__(kThreads, 1)
    gdr_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmO, ChunkArgs a) {
  using Lay = Cfg<PC>;
  constexpr int kStages = Lay::kStages;
  constexpr uint32_t kGateBytes = Lay::kGateBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int H = a.H;
  // Dense: sequence b is row b of the [B, T, H, d] tensors.  Packed
  // (cu_seqlens): sequence b is tokens [cu[b], cu[b + 1]) of row 0 of the
  // [1, total, H, d] tensors.  tb: its first token, bt: its row, T: its
  // length (clamped into the tensor).
  int tb = 0, bt = b, T = a.T;
  if (a.cu_seqlens) {
    const int s0 = min(max(a.cu_seqlens[b], 0), a.T);
    const int s1 = min(max(a.cu_seqlens[b + 1], s0), a.T);
    tb = s0;
    bt = 0;
    T = s1 - s0;
  } else if (a.seg_n > 0) {  // segment b % seg_n of sequence b / seg_n, whole chunks
    const int b0 = b / a.seg_n, p = b % a.seg_n, nc = (a.seg_T + C - 1) / C;
    const int c0 = (int)((long long)p * nc / a.seg_n);
    const int c1 = (int)((long long)(p + 1) * nc / a.seg_n);
    tb = b0 * a.seg_T + c0 * C;
    bt = 0;
    T = min(c1 * C, a.seg_T) - c0 * C;
  }
  const int n = (T + C - 1) / C;

  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::BAR);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lay::MISC + 4);
  float *AF = reinterpret_cast<float *>(sm + Lay::AF);
  // gate vectors of chunk c (one set per K/Q stage)
  auto gate_slot = [&](int c) {
    return reinterpret_cast<float *>(sm + Lay::GS + (c % kStages) * kGateBytes);
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_FULL + s], 1);
      mbar_init(&bars[B_EMPTY + s], 1);
    }
    mbar_init(&bars[B_VFULL], 1);
    mbar_init(&bars[B_VEMPTY], 1);
    mbar_init(&bars[B_D1F], 1);
    mbar_init(&bars[B_D1E], 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_TRDY + s], 4);
      mbar_init(&bars[B_UF + s], 1);
      mbar_init(&bars[B_OE + s], 4);
    }
    mbar_init(&bars[B_ZF], 1);
    mbar_init(&bars[B_ZR], 4);
    mbar_init(&bars[B_VPF], 1);
    mbar_init(&bars[B_VPR], 4);
    mbar_init(&bars[B_SF], 1);
    mbar_init(&bars[B_OF], 1);
    mbar_init(&bars[B_SBR], 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_PE + s], 1);
      mbar_init(&bars[B_TPE + s], 1);
    }
    mbar_init(&bars[B_FIN], 1);
    mbar_init(&bars[B_FIN2], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&bars[B_SCALED + s], 2);
    for (int s = 0; s < 4; ++s) mbar_init(&bars[B_GF + s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Both T and both T' tiles start at zero: their blocks above the block
  // diagonal are never written afterwards.  Additive writes (ADD): T = I for
  // good (in both T tiles, or both T' tiles that per-channel gates use for
  // T), so that the U MMA yields V'^T = V^T.
  for (uint32_t off = 16 * tid; off < (PC ? 2 : 4) * kTileBytes; off += 16 * kThreads) {
    uint4 z = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t tile = off / kTileBytes, row = (off % kTileBytes) / 128;
    if (ADD && tile < 2 && ((off % 128) / 16 ^ (row & 7)) == row / 8) {
      // this 16-byte chunk holds columns 8 (row / 8) .. + 7 of its row: the
      // diagonal element is number row % 8 (bf16 1.0 = 0x3f80)
      const uint32_t e = row & 7, one = 0x3f80u << (16 * (e & 1));
      (&z.x)[e >> 1] = one;
    }
    *reinterpret_cast<uint4 *>(sm + Lay::T + off) = z;
  }
  if (PC) {  // per-channel gates: the scalar gate vectors are constants
    for (int i = tid; i < kStages * 256; i += kThreads) {
      float *gv = reinterpret_cast<float *>(sm + Lay::GS + (i >> 8) * kGateBytes);
      const int k = i & 255;
      gv[k] = k < 64 ? 0.f : 1.f;  // gc = 0; e^{gc}, e^{-gc}, e^{gc_last - gc} = 1
    }
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;
  const uint32_t lane_base = tm + ((uint32_t)((warp & 3) * 32) << 16);

  if (n == 0) {
    // ================================================================ empty packed sequence
    if (warp < 4 && a.S_T) {  // S_T = S0 (or 0); row i of the state per thread
      const float4 *src = a.S0 ? reinterpret_cast<const float4 *>(a.S0 + ((size_t)bh * DV + tid) * DK)
                               : nullptr;
      float4 *dst = reinterpret_cast<float4 *>(a.S_T + ((size_t)bh * DV + tid) * DK);
      for (int e = 0; e < DK / 4; ++e) dst[e] = src ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else if (warp == kProducerWarp) {
    // ================================================================ K/Q producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
    }
    int last_issued[3] = {-1, -1, -1};  // latest chunk loaded into each stage
    int gate_req[2] = {0, 0};              // PC: latest chunk of gate rows requested, per half
    if (PC && lane == 0) {  // this warp's gate rows of chunk 0
      float *gt = reinterpret_cast<float *>(sm + Lay::GT);
      mbar_arrive_expect_tx(&bars[B_GF + 0], 32 * 64 * 4);
      tma_load_4d(gt, &tmG, &bars[B_GF + 0], 0, h, tb, bt);
      mbar_arrive_expect_tx(&bars[B_GF + 1], 32 * 64 * 4);
      tma_load_4d(gt + 32 * 64, &tmG, &bars[B_GF + 1], 0, h, tb + 32, bt);
    }
    // Scalar gates: the state group's scale sequence, replayed with the same
    // fp32 operations: sig = the scale of S_b for the chunk being produced.
    float sig = 1.f;
    // Scalar gates of chunk j into its stage's vectors (prologue: g and
    // beta arrive as logits).
    auto gates = [&](int j) {
      const int t0 = j * C;
      float gl0 = 0.f, gl1 = 0.f, b0 = 0.f, b1 = 0.f;
      const size_t tok = ((size_t)bt * a.T + tb + t0 + lane) * H + h;
      const float gsc = PRO ? a.gate_scale[h] : 0.f;
      if (t0 + lane < T) {
        gl0 = PRO ? -gsc * softplus_f(a.g[tok]) : a.g[tok];
        if (!ADD) b0 = PRO ? sigmoid_f(a.beta[tok]) : a.beta[tok];
      }
      if (t0 + lane + 32 < T) {
        gl1 = PRO ? -gsc * softplus_f(a.g[tok + (size_t)32 * H]) : a.g[tok + (size_t)32 * H];
        if (!ADD) {
          const float bl = a.beta[tok + (size_t)32 * H];
          b1 = PRO ? sigmoid_f(bl) : bl;
        }
      }
      write_scalar_gates(gate_slot(j), gl0, gl1, b0, b1, lane, j, sig);
    };
    for (int c = 0; c < n; ++c) {
      const int s = c % kStages;
      if (c >= kStages &&
          !wait_or_abort(&bars[B_EMPTY + s], ((c / kStages) - 1) & 1, abort_flag))
        break;
      // Testing hook: this chunk's load is never issued, so its consumers'
      // bounded waits run out and the kernel unwinds (no trap, no hang).
      if (c == a.skip_stage_chunk) continue;
      const int t0 = c * C;
      // The K/Q loads go out first; the phase's one arrival follows once the
      // gate vectors are written, so whoever sees the phase sees both.
      if (lane == 0) {
        uint64_t *fb = &bars[B_FULL + s];
        mbar_expect_tx(fb, kKQTx);
        uint8_t *kq = sm + Lay::KQ + s * 4 * kTileBytes;
        tma_load_4d(kq + 0 * kTileBytes, &tmK, fb, 0, h, tb + t0, bt);
        tma_load_4d(kq + 1 * kTileBytes, &tmQ, fb, 0, h, tb + t0, bt);
        tma_load_4d(kq + 2 * kTileBytes, &tmK, fb, 64, h, tb + t0, bt);
        tma_load_4d(kq + 3 * kTileBytes, &tmQ, fb, 64, h, tb + t0, bt);
      }
      last_issued[s] = c;
      float *gv = gate_slot(c);
      if (PC && !ADD) {  // beta only; each scaling warp loads its own gate rows
        const size_t tok = ((size_t)bt * a.T + tb + t0 + lane) * H + h;
        gv[kGateBeta + lane] = t0 + lane < T ? a.beta[tok] : 0.f;
        gv[kGateBeta + lane + 32] = t0 + lane + 32 < T ? a.beta[tok + (size_t)32 * H] : 0.f;
      }
      if (!PC) gates(c);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_FULL + s]);
      if (PC) {  // channels 0-63 of this stage's per-channel scaling
        if (!warp_wait(&bars[B_FULL + s], (c / kStages) & 1, abort_flag, lane)) break;
        float *gt = reinterpret_cast<float *>(sm + Lay::GT);
        const int r = scale_channels(sm + Lay::KQ + s * 4 * kTileBytes,
                                     sm + Lay::KH + s * 2 * kTileBytes, gt, gt + 32 * 64,
                                     &bars[B_GF], c & 1, &tmG, h, bt,
                                     c + 1 < n ? tb + t0 + C : -1, T - t0, gv, 0, lane,
                                     abort_flag, a.status);
        if (c + 1 < n && r >= 1) gate_req[0] = c + 1;
        if (c + 1 < n && r == 2) gate_req[1] = c + 1;
        if (r < 2) break;
        fence_proxy_async_smem();
        warp_arrive(&bars[B_SCALED + (c & 1)]);
      }
    }
    // Loads still in flight after an abort land before the CTA exits (a
    // phase that has already completed passes at once).
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        const int c = last_issued[s];
        if (c >= 0) drain_wait(&bars[B_FULL + s], (c / kStages) & 1);
      }
      if (PC) {
        drain_wait(&bars[B_GF + 0], gate_req[0] & 1);
        drain_wait(&bars[B_GF + 1], gate_req[1] & 1);
      }
    }
  } else if (warp == kVWarp && PC) {
    // ================================================================ V producer + PC scaling
    float *gt = reinterpret_cast<float *>(sm + Lay::GT) + 2 * 32 * 64;  // this warp's rows
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bars[B_GF + 2], 32 * 64 * 4);
      tma_load_4d(gt, &tmG, &bars[B_GF + 2], 64, h, tb, bt);
      mbar_arrive_expect_tx(&bars[B_GF + 3], 32 * 64 * 4);
      tma_load_4d(gt + 32 * 64, &tmG, &bars[B_GF + 3], 64, h, tb + 32, bt);
    }
    int last = -1, gate_req[2] = {0, 0};
    for (int c = 0; c < n; ++c) {
      const int s = c % kStages;
      if (!warp_wait(&bars[B_FULL + s], (c / kStages) & 1, abort_flag, lane)) break;
      float *gv = reinterpret_cast<float *>(sm + Lay::GS + s * kGateBytes);
      const int r = scale_channels(sm + Lay::KQ + s * 4 * kTileBytes,
                                   sm + Lay::KH + s * 2 * kTileBytes, gt, gt + 32 * 64,
                                   &bars[B_GF + 2], c & 1, &tmG, h, bt,
                                   c + 1 < n ? tb + (c + 1) * C : -1, T - c * C, gv, 64, lane,
                                   abort_flag, a.status);
      if (c + 1 < n && r >= 1) gate_req[0] = c + 1;
      if (c + 1 < n && r == 2) gate_req[1] = c + 1;
      if (r < 2) break;
      fence_proxy_async_smem();
      warp_arrive(&bars[B_SCALED + (c & 1)]);
      if (c >= 1 && !warp_wait(&bars[B_VEMPTY], (c - 1) & 1, abort_flag, lane)) break;
      if (lane == 0) {
        uint8_t *vv = sm + Lay::V;
        if (a.zero_v) {  // v taken as zero: the phase completes with no load
          mbar_arrive(&bars[B_VFULL]);
        } else {
          mbar_arrive_expect_tx(&bars[B_VFULL], kVTx);
          tma_load_4d(vv, &tmV, &bars[B_VFULL], 0, h, tb + c * C, bt);
          tma_load_4d(vv + kTileBytes, &tmV, &bars[B_VFULL], 64, h, tb + c * C, bt);
        }
      }
      __syncwarp();
      last = c;
    }
    if (lane == 0 && last >= 0) drain_wait(&bars[B_VFULL], last & 1);
    if (lane == 0) {
      drain_wait(&bars[B_GF + 2], gate_req[0] & 1);
      drain_wait(&bars[B_GF + 3], gate_req[1] & 1);
    }
  } else if (warp == kVWarp) {
    // ================================================================ V producer
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      int last = -1;
      for (int c = 0; c < n; ++c) {
        if (c >= 1 && !wait_or_abort(&bars[B_VEMPTY], (c - 1) & 1, abort_flag)) break;
        uint8_t *vv = sm + Lay::V;
        if (a.zero_v) {  // v taken as zero: the phase completes with no load
          mbar_arrive(&bars[B_VFULL]);
        } else {
          mbar_arrive_expect_tx(&bars[B_VFULL], kVTx);
          tma_load_4d(vv, &tmV, &bars[B_VFULL], 0, h, tb + c * C, bt);
          tma_load_4d(vv + kTileBytes, &tmV, &bars[B_VFULL], 64, h, tb + c * C, bt);
        }
        last = c;
      }
      if (last >= 0) drain_wait(&bars[B_VFULL], last & 1);
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ state-side MMAs
    if (lane == 0) {
      const uint32_t a_kq = smem_u32(sm + Lay::KQ), a_tp = smem_u32(sm + Lay::TP);
      const uint32_t a_p = smem_u32(sm + Lay::P);
      const uint32_t a_kh = smem_u32(sm + Lay::KH), a_v = smem_u32(sm + Lay::V);
      const uint32_t a_t = smem_u32(sm + Lay::T);
      auto W = [&](int slot, uint32_t parity) {
        const bool ok = wait_or_abort(&bars[slot], parity, abort_flag);
        tc_fence_after();
        return ok;
      };
      // Each barrier completes once per chunk (per buffer for PE / TPE) and
      // is waited on by parity, so no arrival may run two phases ahead of
      // its waiter: every producer of a phase first depends, directly or
      // through this thread's program order, on its consumer's previous one.
      bool ok = true;
      for (int c = 0; c < n && ok; ++c) {
        const uint32_t ph = c & 1;
        const int st = c % kStages;
        const uint32_t kq = a_kq + st * 4 * kTileBytes;
        // Z = S_b K^T and O_a = S_b Q^T, their k-steps interleaved: two
        // independent accumulators share the tensor pipe while each waits on
        // its own previous k-step.  O_a goes to buffer c % 2, free once the
        // epilogue has read chunk c - 2's O.  The SF commit below also covers
        // these last reads of S_b (the state group overwrites S_b once SF
        // completes).  (ADD: no correction; no Z.)
        if (!(ok = W(B_SBR, ph) && W(B_FULL + st, (c / kStages) & 1))) break;
        // (segment passes that write no o skip O_a and O_b altogether)
        const bool wo = a.write_o != 0;
        if (wo && c >= 2 && !(ok = W(B_OE + (c & 1), ((c >> 1) - 1) & 1))) break;
        const uint32_t tmo = tm + ((c & 1) ? TM_O1 : TM_O0);
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = kq + (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          if (!ADD)
            mma_bf16_ts(tm + TM_Z, tm + TM_SB + 8 * kk, sdesc_sw128(koff, 16, 1024), ID_N64,
                        kk > 0);
          if (wo)
            mma_bf16_ts(tmo, tm + TM_SB + 8 * kk, sdesc_sw128(koff + kTileBytes, 16, 1024),
                        ID_N64, kk > 0);
        }
        mma_commit(&bars[B_ZF]);
        // U^T = V^T T^T into the V' accumulator, once T of the chunk is
        // written and V has landed (the previous V' was converted: its VPR
        // wait precedes in this thread).  T buffer c % 2 (PC: T is in the T'
        // buffer).
        if (!(ok = W(B_TRDY + (c & 1), (c >> 1) & 1) && W(B_VFULL, ph))) break;
        {
          const uint32_t tt = (PC ? a_tp : a_t) + (c & 1) * kTileBytes;
          if (STASH) {  // backward stash: this chunk's T (map in tmO's slot)
            tma_store_3d(&tmO, sm + Lay::T + (c & 1) * kTileBytes, 0, 0, bh * n + c);
            tma_store_commit();
            tma_store_wait_read0();  // read before the prep group may rewrite the buffer
          }
          if (!a.zero_v) {  // (v taken as zero: U = 0, the V' MMA starts the accumulator)
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(tm + TM_UV, sdesc_sw128(a_v + kk * 2048, kTileBytes, 1024),
                          sdesc_sw128(tt + kk * 32, 16, 1024), ID_U, kk > 0);
          }
          mma_commit(&bars[B_UF + (c & 1)]);  // T read: the prep group may write chunk c + 2's
          mma_commit(&bars[B_VEMPTY]);  // V read
        }
        // V'^T = U^T + Z (-T')^T, or (-Z) T'^T  (ADD: V'^T = U^T = V^T)
        if (!ADD) {
          if (!(ok = W(B_ZR, ph))) break;
          const uint32_t tp = a_tp + (c & 1) * kTileBytes;
          const uint32_t acc0 = a.zero_v ? 0u : 1u;
#pragma unroll 1
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tm + TM_UV, tm + TM_Z + 8 * kk, sdesc_sw128(tp + kk * 32, 16, 1024),
                        ID_N64, kk > 0 ? 1u : acc0);
        }
        mma_commit(&bars[B_VPF]);
        if (!ADD) mma_commit(&bars[B_TPE + (c & 1)]);
        // S_tmem += (V'^T decayed / sigma) K ;  O_b = V'^T P^T, with the bf16
        // copies of V'^T in TMEM as A (PC: the plain copy serves both)
        if (!(ok = W(B_VPR, ph))) break;
        // B = K (MN-major); PC: K^ of the stage
        const uint32_t kb = PC ? a_kh + st * 2 * kTileBytes : kq;
        const uint32_t kb_lbo = PC ? kTileBytes : 2 * kTileBytes;
        const uint32_t vpd = tm + TM_UV + (PC ? 0 : 32);
#pragma unroll 1
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tm + TM_S, vpd + 8 * kk, sdesc_sw128(kb + kk * 2048, kb_lbo, 1024), ID_S,
                      1);
        mma_commit(&bars[B_SF]);
        // O_b accumulated onto the scaled O_a (its scaling precedes the
        // state group's VPR arrival)
        const uint32_t pp = a_p + (c & 1) * kTileBytes;
        if (wo) {
#pragma unroll 1
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmo, tm + TM_UV + 8 * kk, sdesc_sw128(pp + kk * 32, 16, 1024), ID_N64,
                        1);
          mma_commit(&bars[B_OF]);
        }
        mma_commit(&bars[B_PE + (c & 1)]);
        mma_commit(&bars[B_EMPTY + st]);
      }
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(&bars[B_FIN]);
      drain_wait(&bars[B_FIN], 0);
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp == kPrepMmaWarp) {
    // ================================================================ prep-side MMAs
    if (lane == 0) {
      const uint32_t a_kq = smem_u32(sm + Lay::KQ), a_kh = smem_u32(sm + Lay::KH);
      auto W = [&](int slot, uint32_t parity) {
        const bool ok = wait_or_abort(&bars[slot], parity, abort_flag);
        tc_fence_after();
        return ok;
      };
      // chunk c's operands ready: K/Q landed, or (PC) scaled
      auto ready = [&](int c) {
        return PC ? W(B_SCALED + (c & 1), (c >> 1) & 1)
                  : W(B_FULL + c % kStages, (c / kStages) & 1);
      };
      auto issue_d1 = [&](int c) {  // D1 = [K; Q] K^T   (PC: [K~; Q~] K^T)
        const uint32_t kq = a_kq + (c % kStages) * 4 * kTileBytes;
        const uint32_t kh = a_kh + (c % kStages) * 2 * kTileBytes;
#pragma unroll 1
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 2 * kTileBytes + (kk & 3) * 32;
          const uint32_t boff = PC ? kh + (kk >> 2) * kTileBytes + (kk & 3) * 32 : kq + off;
          mma_bf16_ss(tm + TM_D1, sdesc_sw128(kq + off, 16, 1024), sdesc_sw128(boff, 16, 1024),
                      ID_D1, kk > 0);
        }
        mma_commit(&bars[B_D1F]);
      };
      // D1 of chunk c + 1 goes out as soon as the prep group has read D1 of
      // chunk c and the chunk's operands are ready.
      bool ok = ready(0);
      if (ok) issue_d1(0);
      for (int c = 0; c + 1 < n && ok; ++c) {
        if (!(ok = W(B_D1E, c & 1) && ready(c + 1))) break;
        issue_d1(c + 1);
      }
      mma_commit(&bars[B_FIN2]);
      drain_wait(&bars[B_FIN2], 0);
      if (!ok) atomicOr(a.status, kStatusTimeout);
    }
  } else if (warp >= 4 && warp < 8) {
    // ================================================================ prep group
    const int pt = tid - 128, rl = pt;
    const int lrow = rl;
    (void)lrow;
    constexpr uint32_t kBar = 3;
    bool ok = true;
    for (int c = 0; c < n; ++c) {
      const int st = c % kStages;
      const uint32_t ph = c & 1;
      const float *gv = gate_slot(c);
      const float *gcv = gv + kGateGc, *egv = gv + kGateEg, *iegv = gv + kGateIeg;
      const float *bs = gv + kGateBeta;
      // This warp's waits, probed together: the stage, D1, this P buffer
      // free (O_b of chunk c - 2), and for the warps writing A (rows 0-63)
      // every strip of the previous chunk done reading AF (TRDY counts all
      // four prep warps; the P warps probe D1 again in its place).
      // (ADD: no A, so no wait on AF)
      const bool a_rows = !ADD && pt < 64;
      bool bad = !wait_all<4>({&bars[B_FULL + st], &bars[B_D1F],
                               &bars[B_PE + (c & 1)],
                               a_rows ? &bars[B_TRDY + ((c - 1) & 1)] : &bars[B_D1F]},
                              {uint32_t((c / kStages) & 1), ph, uint32_t(((c >> 1) - 1) & 1),
                               a_rows ? uint32_t(((c - 1) >> 1) & 1) : ph},
                              abort_flag);
      if (PRO) {
        // Token norms: 1 / |k| into Rk and folded into the vectors that meet
        // K (Ieg, Egl in place, SEgK = SEg rk), 1 / |q| into Rq and SEgQ =
        // SEg rq.  Thread pt sums half a Q row (token pt / 2, channels
        // 64 (pt % 2) ..); the A rows' threads read their own |k|^2 off D1.
        // Nothing here is skipped on a failed wait: the loads stay in
        // bounds and the shuffle needs every lane; only the writes are.
        float *gw = gate_slot(c);
        const uint8_t *kq = sm + Lay::KQ + st * 4 * kTileBytes;
        float sq = row_sumsq_half(kq + (1 + 2 * (pt & 1)) * kTileBytes + (pt >> 1) * 128, lane);
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        tc_fence_after();
        if (rl < 64) {  // warps 4, 5: D1[rl][rl] is column lane of half rl / 32
          float x[32];
          tmem_ld32(lane_base + TM_D1 + 32 * (rl >> 5), x);
          const float rk = (a.norm_qk & 2) ? rsqrtf(pick_lane(x, lane) + kNormEps) : 1.f;
          if (!bad) {
            gw[kGateRk + rl] = rk;
            gw[kGateSEgK + rl] = gw[kGateSEg + rl] * rk;
            gw[kGateIeg + rl] *= rk;
            gw[kGateEgl + rl] *= rk;
          }
        }
        if (!bad && (pt & 1) == 0) {
          const float rq = (a.norm_qk & 1) ? rsqrtf(sq + kNormEps) : 1.f;
          gw[kGateRq + (pt >> 1)] = rq;
          gw[kGateSEgQ + (pt >> 1)] = gw[kGateSEg + (pt >> 1)] * rq;
        }
        // The group's norms are in; the state group waits for them on the
        // stage's norm barrier.
        if (!group_any(kBar, bad) && pt == 0) mbar_arrive(&bars[B_NORM + st]);
      }
      if (!bad && (!ADD || rl >= 64) && (rl < 64 || a.write_o)) {
        const bool factored = -gcv[63] < kSafeDecay;
        // ---- A (lanes 0-63) and P (lanes 64-127) from D1, 32 columns at a time
        tc_fence_after();
#pragma unroll 1
        for (int hp = 0; hp < 2; ++hp) {
          const int r = rl & 63;
          const float gr = gcv[r];
          // (prologue: the row's 1 / |k| or 1 / |q| as well)
          const float br = (rl < 64 ? bs[r] : 1.f) *
                           (PRO ? gv[(rl < 64 ? kGateRk : kGateRq) + r] : 1.f);
          const float fr = br * egv[r];
          float x[32];
          tmem_ld32(lane_base + TM_D1 + 32 * hp, x);
          DBG_ROW(32 * hp, 64, x);
          const int lim = r + 1 - 32 * hp;  // P: s <= r
          // The decay form is chosen once per chunk, outside the unrolled
          // loops (a branch inside them costs even when it is never taken).
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
          } else {  // rare: chunks whose total decay is beyond e^{-80}
#pragma unroll
            for (int s4 = 0; s4 < 8; ++s4) {
              const float4 gg = *reinterpret_cast<const float4 *>(gcv + 32 * hp + 4 * s4);
              // (prologue: the columns' 1 / |k|, which Ieg carries on the
              // factored path)
              const float4 rc = PRO ? *reinterpret_cast<const float4 *>(gv + kGateRk + 32 * hp +
                                                                        4 * s4)
                                    : make_float4(1.f, 1.f, 1.f, 1.f);
              dvs[4 * s4 + 0] = br * __expf(gr - gg.x) * rc.x;
              dvs[4 * s4 + 1] = br * __expf(gr - gg.y) * rc.y;
              dvs[4 * s4 + 2] = br * __expf(gr - gg.z) * rc.z;
              dvs[4 * s4 + 3] = br * __expf(gr - gg.w) * rc.w;
            }
          }
          if (rl < 64) {
            // A is not masked: what lands at or above its diagonal is never
            // read (the diagonal blocks are replaced by their inverses before
            // any other use, the blocks above them are not used).
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= dvs[e];
            float4 *dst = reinterpret_cast<float4 *>(AF + r * LDA + 32 * hp);
#pragma unroll
            for (int s4 = 0; s4 < 8; ++s4)
              dst[s4] = make_float4(x[4 * s4], x[4 * s4 + 1], x[4 * s4 + 2], x[4 * s4 + 3]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = (e < lim) ? x[e] * dvs[e] : 0.f;
            st_row32_sw128(sm + Lay::P + (c & 1) * kTileBytes, r, hp, x);
          }
        }
        if (rl >= 64) fence_proxy_async_smem();  // P is read by the tensor core
      }
      if (!bad) {
        tc_fence_before();
        warp_arrive(&bars[B_D1E]);  // this thread's D1 reads are done
      }
      if (ADD) {
        // T = I throughout: only P is handed on, once U of chunk c - 2 has
        // completed (which keeps TRDY buffer c % 2 within one phase of its
        // waiter).
        bad = bad || !warp_wait(&bars[B_UF + (c & 1)], ((c >> 1) - 1) & 1, abort_flag, lane);
        if (group_any(kBar, bad)) { ok = false; break; }
        warp_arrive(&bars[B_TRDY + (c & 1)]);
        continue;
      }
      // ---- Y = (I + A)^{-1} -> T, T' (buffers c % 2): free once U (T) and
      //      V' (T') of chunk c - 2 have completed.
      uint8_t *tpc = sm + Lay::TP + (c & 1) * kTileBytes;
      const TOut to{PC ? tpc : sm + Lay::T + (c & 1) * kTileBytes, tpc, bs,
                    PC ? egv : gv + (PRO ? kGateSEgK : kGateSEg)};
      bad = bad || !wait_all<2>({&bars[B_UF + (c & 1)], &bars[B_TPE + (c & 1)]},
                                {uint32_t(((c >> 1) - 1) & 1), uint32_t(((c >> 1) - 1) & 1)},
                                abort_flag);
      if (!bad && rl < 64) {  // the warps that wrote A invert its diagonal blocks
        __syncwarp();
        invert_diag(AF, to, rl >> 5, lane);
      }
      // A and every D_bb complete in AF; the group agrees on failure.
      if (group_any(kBar, bad)) { ok = false; break; }
      diag_to_t<!PC>(AF, to, pt);
      {
        float *ysc = reinterpret_cast<float *>(sm + Lay::SCR);  // [2][16][16]
        float *wscr = ysc + 512;                                 // 4 warps x 2 x [16][8]
        invert_level1<!PC>(AF, ysc, wscr, to, pt);
        if (group_any(kBar, false)) { ok = false; break; }  // Y_10, Y_32 in ysc
        invert_level2<!PC>(AF, ysc, wscr, to, pt);
      }
      fence_proxy_async_smem();
      warp_arrive(&bars[B_TRDY + (c & 1)]);  // this thread's T, T', P writes are done
    }
    if (!ok && pt == 0) atomicOr(a.status, kStatusTimeout);
  } else if (warp < 4) {
    // ================================================================ state group
    const int i = tid;  // TMEM lane = value channel
    const int lrow = i;
    (void)lrow;
    bool ok = true;
    // Gate factors of chunk c for this group: e^{gc_r} and e^{gc_last - gc_r}
    // into its SVEC slot; returns the chunk's total decay e^{gc_last}.
    // Every warp writes the same values and reads them after its own writes
    // (no group barrier).  A warp cannot run a whole chunk ahead of another:
    // the four-warp barriers it waits for need the other warps' arrivals.
    // With additive writes it can, however, write chunk c + 2's copy while
    // another warp still reads chunk c's in its O epilogue (nothing ties V'
    // of chunk c + 1 to that epilogue; otherwise the Z hand-off of chunk
    // c + 1 does), hence three slots there, two otherwise.
    auto svec = [&](int c) {
      return sm + Lay::SVEC + (ADD ? c % 3 : c & 1) * Lay::kSvecBytes;
    };
    auto chunk_vectors = [&](int c, float &dl) -> bool {
      // (prologue: the stage's vectors are final once its norms are folded in)
      const bool got =
          PC ? warp_wait(&bars[B_SCALED + (c & 1)], (c >> 1) & 1, abort_flag, lane)
             : warp_wait(&bars[(PRO ? B_NORM : B_FULL) + c % kStages], (c / kStages) & 1,
                         abort_flag, lane);
      if (!got) return false;
      // The stage can be refilled while this chunk's O epilogue still runs,
      // so the group keeps its own copy of e^{gc} and e^{gc_last - gc}.
      float *sv = reinterpret_cast<float *>(svec(c));
      const float *gv = gate_slot(c);
      // O epilogue: sigma e^{gc} (prologue: times the token's 1 / |q|)
      constexpr int kEg = PC ? kGateEg : (PRO ? kGateSEgQ : kGateSEg);
      sv[kSvEg + lane] = gv[kEg + lane];
      sv[kSvEg + lane + 32] = gv[kEg + lane + 32];
      if (PC || c == 0) {  // scalar gates, c >= 1: written with 1 / sigma by the pass
        sv[kSvEgl + lane] = gv[kGateEgl + lane];
        sv[kSvEgl + lane + 32] = gv[kGateEgl + lane + 32];
      }
      if (PC) {  // per-column factors (the previous chunk's stay in the other slot)
#pragma unroll
        for (int k = lane; k < 128; k += 32) {
          sv[kSvEm + k] = gv[kGateEm + k];
          sv[kSvEgm + k] = gv[kGateEgm + k];
        }
      }
      __syncwarp();
      dl = gv[kGateEg + 63];
      return true;
    };
    // PC: S_tmem <- S_tmem Diag(f1) Diag(f2) and S_b = bf16 of the result
    // (per-column factors, broadcast from shared memory).  f1 = e^{gc_last - m}
    // of the chunk just done takes S_tmem to the true state, f2 = e^{m} of the
    // next chunk to its frame; the two are applied one after the other because
    // their product can underflow where neither frame does.
    auto pass_vec = [&](const float *fv, const float *fv2) {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float x[32];
        tmem_ld32(lane_base + TM_S + 32 * q, x);
        const float4 *f4 = reinterpret_cast<const float4 *>(fv + 32 * q);
        const float4 *g4 = reinterpret_cast<const float4 *>(fv2 + 32 * q);
#pragma unroll
        for (int s4 = 0; s4 < 8; ++s4) {
          const float4 f = f4[s4], f2 = g4[s4];
          x[4 * s4] = x[4 * s4] * f.x * f2.x;
          x[4 * s4 + 1] = x[4 * s4 + 1] * f.y * f2.y;
          x[4 * s4 + 2] = x[4 * s4 + 2] * f.z * f2.z;
          x[4 * s4 + 3] = x[4 * s4 + 3] * f.w * f2.w;
        }
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        tmem_st16u(lane_base + TM_SB + 16 * q, u);
        tmem_st16(lane_base + TM_S + 32 * q, *reinterpret_cast<float(*)[16]>(x));
        tmem_st16(lane_base + TM_S + 32 * q + 16, *reinterpret_cast<float(*)[16]>(x + 16));
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&bars[B_SBR]);
    };
    // S_b = bf16(S_tmem) for the chunk's MMAs (true state / sigma: T' and
    // the O epilogue carry sigma).  While sigma * dl (dl: the chunk's decay)
    // stays above the floor only sigma changes; otherwise (fold) S_tmem <-
    // f S_tmem with f = sigma * dl and sigma restarts at 1.
    // (backward stash: xst = row i of the next chunk's X0, xs = sigma, the
    // scale that takes S_tmem to the true state)
    auto pass_from_tmem = [&](bool fold, float f, uint4 *xst, float xs) {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float x[32];
        tmem_ld32(lane_base + TM_S + 32 * q, x);
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        tmem_st16u(lane_base + TM_SB + 16 * q, u);
        if (xst) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            xst[4 * q + e] = make_uint4(pack_bf16(xs * x[8 * e], xs * x[8 * e + 1]),
                                        pack_bf16(xs * x[8 * e + 2], xs * x[8 * e + 3]),
                                        pack_bf16(xs * x[8 * e + 4], xs * x[8 * e + 5]),
                                        pack_bf16(xs * x[8 * e + 6], xs * x[8 * e + 7]));
        }
        if (fold) {  // rare: write back S_tmem * f
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= f;
          tmem_st16(lane_base + TM_S + 32 * q, *reinterpret_cast<float(*)[16]>(x));
          tmem_st16(lane_base + TM_S + 32 * q + 16, *reinterpret_cast<float(*)[16]>(x + 16));
        }
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(&bars[B_SBR]);
    };
    // sig: the scale of S_tmem at the next state pass.  1 / the scale after
    // the chunk in flight is applied to that chunk's state update through the
    // group's copy of e^{gc_last - gc}.
    float sig = 1.f;
    {
      float dl;
      if (!chunk_vectors(0, dl)) {
        ok = false;
      } else {
        // S_b = bf16(S0); S_tmem = e^{gc_last} S0; sigma = 1 afterwards.
        // Segment passes: S0 of the first segment of each sequence only
        // (a.s0_seg segments per sequence, S0 indexed by sequence), or the
        // identity (the run that yields a segment's transition).
        const float *s0 = nullptr;
        if (a.S0 && a.s0_seg == 0) {
          s0 = a.S0 + ((size_t)bh * DV + i) * DK;
        } else if (a.S0 && b % a.s0_seg == 0) {
          s0 = a.S0 + (((size_t)(b / a.s0_seg) * H + h) * DV + i) * DK;
        }
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          if (s0) {
            const float4 *s4 = reinterpret_cast<const float4 *>(s0 + 32 * q);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 v = s4[e];
              x[4 * e] = v.x;
              x[4 * e + 1] = v.y;
              x[4 * e + 2] = v.z;
              x[4 * e + 3] = v.w;
            }
          } else {
            const float one = a.s0_identity ? 1.f : 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = (32 * q + e == i) ? one : 0.f;
          }
          if (PC) {  // S Diag(e^{m_0})
            const float *fv = reinterpret_cast<const float *>(sm + Lay::SVEC) + kSvEm + 32 * q;
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= fv[e];
          }
          uint32_t u[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
          tmem_st16u(lane_base + TM_SB + 16 * q, u);
          if (STASH) {  // backward stash: row i of chunk 0's X0 (the start state)
            uint4 *xst = reinterpret_cast<uint4 *>(a.stash_x + (((size_t)bh * n) * DV + i) * DK);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              xst[4 * q + e] = make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
          }
          float y0[16], y1[16];
          const float dl0 = PC ? 1.f : dl;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            y0[e] = x[e] * dl0;
            y1[e] = x[16 + e] * dl0;
          }
          tmem_st16(lane_base + TM_S + 32 * q, y0);
          tmem_st16(lane_base + TM_S + 32 * q + 16, y1);
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(&bars[B_SBR]);
      }
    }
    for (int c = 0; ok && c < n; ++c) {
      const uint32_t ph = c & 1;
      const float *sv = reinterpret_cast<const float *>(svec(c));
      const float *egv = sv + kSvEg, *eglv = sv + kSvEgl;
      const uint32_t tmo = lane_base + ((c & 1) ? TM_O1 : TM_O0);
      // ---- Z (scalar gates: T' is stored negated) or -Z (per-channel gates,
      //      whose T' buffer is T itself) -> bf16 A operand, in place in TMEM
      //      (ZF also covers O_a)
      if (!warp_wait(&bars[B_ZF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      if (!ADD) {
      {
        // both halves are loaded before either is overwritten in place
        float z0[32], z1[32];
        tmem_ld32(lane_base + TM_Z, z0);
        tmem_ld32(lane_base + TM_Z + 32, z1);
        DBG_ROW(16384, 64, z0);
        DBG_ROW(16384 + 32, 64, z1);
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          u[e] = PC ? pack_bf16(-z0[2 * e], -z0[2 * e + 1]) : pack_bf16(z0[2 * e], z0[2 * e + 1]);
        tmem_st16u(lane_base + TM_Z, u);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          u[e] = PC ? pack_bf16(-z1[2 * e], -z1[2 * e + 1]) : pack_bf16(z1[2 * e], z1[2 * e + 1]);
        tmem_st16u(lane_base + TM_Z + 16, u);
        tmem_wait_st();
      }
      tc_fence_before();
      warp_arrive(&bars[B_ZR]);
      }
      // ---- O_a Diag(sigma e^{gc}) in place (fp32), off the chain: the
      //      state group would otherwise wait for V' here.  O_b is then
      //      accumulated onto it.  (PC: the factors are 1, Q~ carries the
      //      decay.)  Stored before the VPR arrival below.
      if (!PC && a.write_o) {
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
          float x[32];
          tmem_ld32(tmo + 32 * q, x);
          const float4 *e4 = reinterpret_cast<const float4 *>(egv + 32 * q);
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 e = e4[s4];
            x[4 * s4] *= e.x;
            x[4 * s4 + 1] *= e.y;
            x[4 * s4 + 2] *= e.z;
            x[4 * s4 + 3] *= e.w;
          }
          tmem_st16(tmo + 32 * q, *reinterpret_cast<float(*)[16]>(x));
          tmem_st16(tmo + 32 * q + 16, *reinterpret_cast<float(*)[16]>(x + 16));
        }
      }
      // ---- V'^T -> its bf16 A operands, in place in TMEM: plain in columns
      //      0-31, decayed to the chunk end / sigma in 32-63 (PC: the plain
      //      copy serves both)
      if (!warp_wait(&bars[B_VPF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      {
        // both halves are loaded before either is overwritten in place
        float x0[32], x1[32];
        tmem_ld32(lane_base + TM_UV, x0);
        tmem_ld32(lane_base + TM_UV + 32, x1);
        DBG_ROW(40960, 64, x0);
        DBG_ROW(40960 + 32, 64, x1);
        uint32_t u[16];
        // (backward stash: row i of V'^T, tokens 0-63)
        uint4 *vst = STASH ? reinterpret_cast<uint4 *>(a.stash_v + (((size_t)bh * n + c) *
                                                                      DV + i) * C)
                           : nullptr;
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x0[2 * e], x0[2 * e + 1]);
        tmem_st16u(lane_base + TM_UV, u);
        if (vst) {
#pragma unroll
          for (int e = 0; e < 4; ++e) vst[e] = make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x1[2 * e], x1[2 * e + 1]);
        tmem_st16u(lane_base + TM_UV + 16, u);
        if (vst) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            vst[4 + e] = make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
        }
        if (!PC) {
          const float4 *e4 = reinterpret_cast<const float4 *>(eglv);
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 e = e4[s4];
            u[2 * s4] = pack_bf16(x0[4 * s4] * e.x, x0[4 * s4 + 1] * e.y);
            u[2 * s4 + 1] = pack_bf16(x0[4 * s4 + 2] * e.z, x0[4 * s4 + 3] * e.w);
          }
          tmem_st16u(lane_base + TM_UV + 32, u);
#pragma unroll
          for (int s4 = 0; s4 < 8; ++s4) {
            const float4 e = e4[8 + s4];
            u[2 * s4] = pack_bf16(x1[4 * s4] * e.x, x1[4 * s4 + 1] * e.y);
            u[2 * s4 + 1] = pack_bf16(x1[4 * s4 + 2] * e.z, x1[4 * s4 + 3] * e.w);
          }
          tmem_st16u(lane_base + TM_UV + 48, u);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      warp_arrive(&bars[B_VPR]);
      // next chunk's gate factors, while the state update runs
      float dl = 1.f;
      if (c + 1 < n && !chunk_vectors(c + 1, dl)) { ok = false; break; }
      // ---- updated S -> S_b for the next chunk, or the final state
      if (!warp_wait(&bars[B_SF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      if (c + 1 < n) {
#ifdef GDR_TC_DEBUG
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          for (int e = 0; e < 32; ++e) x[e] *= sig;
          DBG_ROW(57344 + 32 * q, 128, x);
        }
#endif
        if (PC) {
          pass_vec(sv + kSvEgm, reinterpret_cast<const float *>(svec(c + 1)) + kSvEm);
        } else {
          const float nxt = sig * dl;
          const bool fold = !(nxt >= kScaleFloor);  // also when dl underflows to 0
          pass_from_tmem(fold, nxt,
                         STASH ? reinterpret_cast<uint4 *>(
                                     a.stash_x + (((size_t)bh * n + c + 1) * DV + i) * DK)
                               : nullptr,
                         sig);
          sig = fold ? 1.f : nxt;
          // next chunk's e^{gc_last - gc} / sigma for its update (every warp
          // writes the same values, from the stage, after its own pass)
          const float inv = 1.f / sig;
          const float *gn = gate_slot(c + 1);
          float *svn = reinterpret_cast<float *>(svec(c + 1));
          svn[kSvEgl + lane] = gn[kGateEgl + lane] * inv;
          svn[kSvEgl + lane + 32] = gn[kGateEgl + lane + 32] * inv;
          __syncwarp();
        }
      } else if (a.S_T) {
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float x[32];
          tmem_ld32(lane_base + TM_S + 32 * q, x);
          if (PC) {  // S = S_tmem Diag(e^{gc_last - m})
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= sv[kSvEgm + 32 * q + e];
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] *= sig;
          }
          DBG_ROW(57344 + 32 * q, 128, x);
          float4 *dst = reinterpret_cast<float4 *>(a.S_T + ((size_t)bh * DV + i) * DK + 32 * q);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        }
      }
      // ---- O (= O_a Diag(sigma e^{gc}) + O_b, in buffer c % 2) -> bf16 -> o
      if (!a.write_o) continue;
      if (!warp_wait(&bars[B_OF], ph, abort_flag, lane)) { ok = false; break; }
      tc_fence_after();
      {
        // The warp stages its 32 channels x 64 tokens (bf16, [token][channel],
        // 64-byte rows) in its own quarter of STG, free once the warp's
        // previous store has read it, and one lane stores the box with TMA
        // (rows past T are clipped).  O is read in the 16-lane shape, which gives each
        // thread two adjacent tokens of a channel, so one transposing matrix
        // store writes 8 tokens x 32 channels per warp.
        if (lane == 0) tma_store_wait_read0();  // the previous o store has read STG
        __syncwarp();
        const uint32_t stg = smem_u32(sm + Lay::STG + 4096 * warp);
        // row address of this thread in a matrix store: token 8 k + lane % 8
        // of channel group lane / 8 (matrix j = lane / 8 holds channels
        // 8 j .. 8 j + 7).  The staging tile is 64-byte swizzled (16-byte
        // chunk j of row r at chunk j ^ ((r / 2) % 4), as the TMA store
        // expects), so the 8 rows of a matrix fall in distinct banks.
        const int r8 = lane & 7;
        const uint32_t row_addr = stg + r8 * 64 + 16 * ((lane >> 3) ^ ((r8 >> 1) & 3));
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
          // lanes 0-15 / 16-31 of the warp's quarter, tokens 32 q .. 32 q + 31
          float a0[16], a1[16];
          tmem_ld16x256b_x4(tmo + 32 * q, a0);
          tmem_ld16x256b_x4(tmo + (16u << 16) + 32 * q, a1);
          tmem_wait_ld();
          if (q == 1) {  // every read of this O buffer is done
            tc_fence_before();
            warp_arrive(&bars[B_OE + (c & 1)]);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // tokens 32 q + 8 k + 2 tq, + 1
            const int e = 4 * k;
            stmatrix_x4_trans(row_addr + (4 * q + k) * 512, pack_bf16(a0[e], a0[e + 1]),
                              pack_bf16(a0[e + 2], a0[e + 3]), pack_bf16(a1[e], a1[e + 1]),
                              pack_bf16(a1[e + 2], a1[e + 3]));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int rows = T - c * C;  // valid rows of the chunk
        if ((a.cu_seqlens || a.seg_n > 0) && rows < C) {
          // The last chunk of a packed sequence: the TMA box would run into
          // the next sequence's rows, so the valid rows go out with plain
          // 16-byte stores (chunk j of staging row r sits at j ^ ((r / 2) % 4)).
          if (a.write_o) {
            const uint8_t *st = sm + Lay::STG + 4096 * warp;
            for (int r = lane; r < rows; r += 32) {
              uint4 *dst = reinterpret_cast<uint4 *>(
                  reinterpret_cast<__nv_bfloat16 *>(a.o) +
                  (((size_t)bt * a.T + tb + c * C + r) * H + h) * DV + 32 * warp);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = *reinterpret_cast<const uint4 *>(st + r * 64 + 16 * (j ^ ((r >> 1) & 3)));
            }
          }
        } else if (lane == 0) {
          if (a.write_o)
            tma_store_4d(&tmO, sm + Lay::STG + 4096 * warp, 32 * warp, h, tb + c * C, bt);
          tma_store_commit();
        }
      }
    }
    // stores still reading shared memory or in flight complete before exit
    if (lane == 0) tma_store_wait0();
    if (!ok && lane == 0) atomicOr(a.status, kStatusTimeout);
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

// 4-D map over the output o [B, T, H, d] bf16 for the epilogue's stores:
// box = 64 tokens x 32 channels (one state warp's), 64-byte rows, 64-byte
// swizzle (16-byte chunk j of row r lands at chunk j ^ ((r / 2) % 4)).
bool make_map_out(CUtensorMap *m, void *base, int B, int T, int H, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {32, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D map over the per-channel gate g [B, T, H, d] fp32, box = 32 tokens x
// 64 channels (one scaling warp's half chunk: 256-byte rows, no swizzle).
bool make_map_gate(CUtensorMap *m, const float *base, int B, int T, int H, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)T * H * d * 4};
  cuuint32_t box[4] = {64, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map_stash_t(CUtensorMap *m, void *base, long long nchunks) {
  return tc_map_stash(m, base, nchunks, 64, 64);
}

template <bool PC, bool ADD, bool PRO, bool STASH = false>
cudaError_t launch_variant(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv, const CUtensorMap &mg, const CUtensorMap &mo,
                           cudaStream_t stream) {
  constexpr size_t smem = Cfg<PC>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(gdr_chunk_tc_kernel<PC, ADD, PRO, STASH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gdr_chunk_tc_kernel<PC, ADD, PRO, STASH>
      <<<(unsigned)((size_t)a.B * a.H), kThreads, smem, stream>>>(mq, mk, mv, mg, mo, a);
  return cudaGetLastError();
}

template <bool PC>
cudaError_t launch_pc(const ChunkArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                      const CUtensorMap &mv, const CUtensorMap &mg, const CUtensorMap &mo,
                      cudaStream_t stream) {
  if (a.additive) return launch_variant<PC, true, false>(a, mq, mk, mv, mg, mo, stream);
  if constexpr (!PC) {  // the prologue instance exists for scalar gates only
    if (a.prologue) return launch_variant<false, false, true>(a, mq, mk, mv, mg, mo, stream);
  } else {
    if (a.prologue) return cudaErrorNotSupported;
  }
  return launch_variant<PC, false, false>(a, mq, mk, mv, mg, mo, stream);
}

}  // namespace

bool tc_map_bf16(CUtensorMap *m, const void *base, int B, int T, int H, int d) {
  return make_map(m, base, B, T, H, d);
}

// 3-D map over a per-chunk array [nchunks][rows][cols] bf16 (row-major), box
// 64 columns x 64 rows of one chunk, 128-byte swizzle (the tile layout of
// the tensor-core kernels).
bool tc_map_stash(CUtensorMap *m, const void *base, long long nchunks, int rows, int cols) {
  auto fn = encode_fn();
  if (!fn || nchunks <= 0 || nchunks > 0x7fffffffLL || rows < 64 || cols < 64) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)nchunks};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool chunk_tc_supports(const ChunkArgs &a) {
  return a.bf16 && a.dk == DK && a.dv == DV && a.T > 0 && (size_t)a.B * a.H <= 0x7fffffffu;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream) {
  if (!chunk_tc_supports(a)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mg, mo;
  // Without an output (segment passes) the output map is never used; it is
  // built over q so that it is a valid map.
  // (packed sequences: the tensors are [1, total, H, d]; one CTA per sequence and head)
  const int mb = (a.cu_seqlens || a.seg_n > 0) ? 1 : a.B;
  if (!make_map(&mq, a.q, mb, a.T, a.H, DK) || !make_map(&mk, a.k, mb, a.T, a.H, DK) ||
      !make_map(&mv, a.v, mb, a.T, a.H, DV) ||
      !make_map_out(&mo, a.write_o ? a.o : const_cast<void *>(a.q), mb, a.T, a.H, DV))
    return cudaErrorInvalidValue;
  if (a.stash_t) {  // backward stash (no o): the T tiles go out through the output map's slot
    if (a.per_channel || a.write_o || a.cu_seqlens) return cudaErrorNotSupported;
    if (!make_map_stash_t(&mo, a.stash_t, (long long)a.B * a.H * ((a.T + C - 1) / C)))
      return cudaErrorInvalidValue;
  }
  if (a.stash_t) {
    if (!a.stash_x || !a.stash_v || a.additive || a.prologue) return cudaErrorNotSupported;
    return launch_variant<false, false, false, true>(a, mq, mk, mv, mq, mo, stream);
  }
  if (a.per_channel) {
    if (!make_map_gate(&mg, a.g, mb, a.T, a.H, DK)) return cudaErrorInvalidValue;
    return launch_pc<true>(a, mq, mk, mv, mg, mo, stream);
  }
  return launch_pc<false>(a, mq, mk, mv, mq, mo, stream);  // gate map unused
}

}  // namespace gdr

#ifdef GDR_TC_DEBUG
extern "C" int gdr_debug_set_buffer(float *p, int chunk) {
  if (cudaMemcpyToSymbol(gdr::g_dbg, &p, sizeof p) != cudaSuccess) return 1;
  return cudaMemcpyToSymbol(gdr::g_dbg_chunk, &chunk, sizeof chunk) != cudaSuccess;
}
#endif
