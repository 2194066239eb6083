// Chunked backward of the gated delta rule on the sm_100a tensor cores
// (tcgen05): scalar gate, bf16 q/k/v, d_k = d_v = 128, C = 64.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 5 (the
// chunked form; backpropagation chunked and parallelised with
// recomputation).  Reverse mode through the chunk equations, per chunk,
// written in the state's orientation (S is d_v x d_k; dS = dL/dS):
//
//   forward:  V'^T = U^T - S0 W^T,   O^T = S0 Q~^T + V'^T P^T,
//             S1 = e^{gl} S0 + V'^T K-bar
//             (U = T V, W = T Diag(b) K, K-bar = Diag(e^{gl} / b) K,
//              Q~ = Diag(b) Q, P = tril(Q~ (K / b)^T), b = e^{gc})
//   backward: dV'^T = dO^T P + dS1 K-bar^T
//             dS0   = e^{gl} dS1 + dO^T Q~ - (dV'^T T~) K,   T~ = T Diag(b)
//
// and then, per chunk and in parallel over chunks, the token gradients
// (X0 = S0^T, dX1 = dS1^T, Y = (I + A)^{-1}, T = Y Diag(beta)):
//
//   dP  = tril(dO V'^T)          dW = -dV' X0^T          dT = dV' V^T + dW K~^T
//   dY  = dT Diag(beta)          dA = strict_tril(-Y^T dY Y^T)      dM = Diag(beta) dA
//   dQ~ = dO X0^T + dP K^        dK^ = dP^T Q~ + dM^T K~
//   dK~ = T^T dW + dM K^         dK-bar = V' dX1^T                  dV = T^T dV'
//   dbeta_s = sum_r dT[r][s] Y[r][s] + sum_s' dA[s][s'] M[s][s'],  M = K~ K^^T
//   then through K~ = K b, K^ = K / b, Q~ = Q b, K-bar = K e^{gl} / b and
//   the log-space cumsum of the gates (reverse cumsum of the gate gradient).
//
// Three launches:
//   1. the forward kernel again, stashing per chunk the start state X0, V'^T
//      and T in bf16 (no o);
//   2. this file's state kernel: one CTA per (b, h), chunks in reverse, dS
//      in fp32 in TMEM; it stashes dS1 and dV'^T per chunk and writes dS0;
//   3. this file's gradient kernel: one CTA per chunk and head.
// Every product runs on tcgen05 (kind::f16, bf16 operands, fp32
// accumulators in TMEM), written straight-line: four warps, one thread
// issuing the MMAs, each result read back by the warps that own its TMEM
// lanes.  No TMA load uses cluster multicast; every wait is bounded.
#include <cudaTypedefs.h>

#include "gdr_internal.cuh"
#include "gdr_tc_util.cuh"

namespace gdr {
namespace {

using namespace sm100;
using namespace tcu;

constexpr int C = 64, D = 128;
constexpr int kStateThreads = 256;  // the reverse state pass
constexpr int kGradThreads = 256;   // the gradient pass
constexpr uint32_t kTile = 8192;             // one 64 x 64 bf16 tile (128-byte swizzle)
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait

// Scale the 8 bf16 of a 16-byte chunk by f (one factor) in place.
__device__ __forceinline__ void scale_chunk(uint8_t *p, float f) {
  uint4 v = *reinterpret_cast<uint4 *>(p);
  uint32_t *w = &v.x;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = unpack_bf16(w[e]);
    w[e] = pack_bf16(x.x * f, x.y * f);
  }
  *reinterpret_cast<uint4 *>(p) = v;
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *m, uint64_t *bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// Bulk copies of contiguous bytes (sizes and addresses multiples of 16):
// shared -> global with a bulk group (this thread waits for its reads of
// shared memory, or for completion), and global -> shared completing on an
// mbarrier's transaction count.
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_load(void *sdst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(sdst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte global -> shared copy through the asynchronous copy unit, the
// commit of this thread's copies, and the wait for them.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Bounded wait of every thread, then a CTA-wide agreement (a thread that
// timed out makes every thread leave together).
__device__ __forceinline__ bool wait_all_threads(uint64_t *bar, uint32_t parity, bool ok) {
  ok = ok && mbar_wait_bounded(bar, parity, kWaitNs);
  return __syncthreads_and(ok) != 0;
}

// Inclusive prefix sum of a chunk's 64 log decays (lane l: rows l, l + 32);
// one warp.  Returns the chunk total.
__device__ __forceinline__ float cumsum64(float &x0, float &x1, int lane) {
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

// ====================================================================== state pass
struct StateArgs {
  const float *g;     // [B, T, H]
  const float *dout;  // [B, T, H, D] fp32
  const float *dST;   // [B, H, D, D] or null
  float *dS0;         // [B, H, D, D] or null
  __nv_bfloat16 *stash_ds;  // [B H n][D][D]: dS1 of every chunk (written)
  __nv_bfloat16 *stash_dv;  // [B H n][D][C]: dV'^T of every chunk (written)
  uint8_t *stash_do;        // [B H n][16 KB]: dO of every chunk, bf16, as the swizzled tiles
  int B, T, H, n;
  unsigned int *status;
};

// Shared memory (bytes from a 1024-byte aligned base): two stages of
// [K_h0|Q_h0|K_h1|Q_h1] and of T (T~ once scaled) so that the next chunk's
// loads run under this one's work, [dO_h0|dO_h1] (bf16), P,
// [K-bar_h0|K-bar_h1], the next chunk's dO in fp32 (asynchronous copies),
// gate vectors, barriers.
constexpr uint32_t R_KQ = 0, R_TT = 8 * kTile, R_DO = 10 * kTile, R_P = 12 * kTile,
                   R_KB = 13 * kTile, R_STG = 15 * kTile, R_VEC = 19 * kTile,  // STG: 32 KB
                   R_BAR = R_VEC + 1024, R_MISC = R_BAR + 64, R_END = R_MISC + 64;
constexpr size_t kStateSmem = R_END + 1024;
// TMEM columns: dS (fp32), its bf16 copy, dV'^T, Zc = dV'^T T~, D1 = [K; Q] K^T
constexpr uint32_t TR_DS = 0, TR_DSB = 128, TR_DVP = 192, TR_ZC = 256, TR_D1 = 320;

__global__ void __launch_bounds__(kStateThreads, 1)
    gdr_bwd_state_kernel(const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmT, StateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  // 8 warps: warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 (value
  // channels) and split each per-lane phase's columns between them (hs)
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, lq = warp & 3, hs = warp >> 2;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H, H = a.H, n = a.n;
  uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + R_BAR), *bar_mma = bar_ld + 2;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + R_MISC);
  float *gcv = reinterpret_cast<float *>(sm + R_VEC);  // [64] cumulative log decay
  float *bv = gcv + 64;                                 // [64] e^{gc}
  float *kbv = gcv + 128;                               // [64] e^{gc_last - gc}
  if (t == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_ld + 1, 1);
    mbar_init(bar_mma, 1);
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
  const uint32_t lb = tm + ((uint32_t)(lq * 32) << 16);  // this warp's 32 lanes
  const int i = lq * 32 + lane;                          // TMEM lane = value channel

  // dS = dL/dS_T (or 0)
#pragma unroll 1
  for (int q = hs; q < 4; q += 2) {
    float x[32];
    const float *src = a.dST ? a.dST + ((size_t)bh * D + i) * D + 32 * q : nullptr;
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = src ? src[e] : 0.f;
    tmem_st32(lb + TR_DS + 32 * q, x);
  }
  tmem_wait_st();

  const uint32_t dq = smem_u32(sm + R_DO);
  const uint32_t pp = smem_u32(sm + R_P), kb = smem_u32(sm + R_KB);
  constexpr uint32_t ID_D1 = idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t ID_DOP = idesc_bf16(128, 64, 1, 1);   // A = dO^T, B = P (both MN-major)
  constexpr uint32_t ID_KB = idesc_bf16(128, 64, 0, 0);    // A = dS1 (TMEM), B = K-bar
  constexpr uint32_t ID_ZC = idesc_bf16(128, 64, 0, 1);    // A = dV'^T (TMEM), B = T~
  constexpr uint32_t ID_DOQ = idesc_bf16(128, 128, 1, 1);  // A = dO^T, B = Q~
  constexpr uint32_t ID_ZK = idesc_bf16(128, 128, 0, 1);   // A = -Zc (TMEM), B = K
  // Chunk c's K, Q and T into stage st by TMA (rows past T read as zero);
  // thread 0 only.  ld_n counts the loads each stage has received.
  int ld_n0 = 0, ld_n1 = 0;
  auto load_tiles = [&](int c, int st) {
    uint64_t *bl = bar_ld + st;
    uint8_t *kqs = sm + R_KQ + st * 4 * kTile;
    const int c0 = c * C;
    mbar_arrive_expect_tx(bl, 5 * kTile);
    tma_load_4d(kqs + 0 * kTile, &tmK, bl, 0, h, c0, b);
    tma_load_4d(kqs + 1 * kTile, &tmQ, bl, 0, h, c0, b);
    tma_load_4d(kqs + 2 * kTile, &tmK, bl, 64, h, c0, b);
    tma_load_4d(kqs + 3 * kTile, &tmQ, bl, 64, h, c0, b);
    tma_load_3d(sm + R_TT + st * kTile, &tmT, bl, 0, 0, bh * n + c);
    if (st) ++ld_n1; else ++ld_n0;
  };
  // Chunk c's dO rows into the fp32 staging area through the asynchronous
  // copy unit: this thread's row t / 2, channel half t % 2 (rows past T are
  // not copied).  Only the thread that copies a row half reads it back.
  auto load_dout = [&](int c) {
    const int c0 = c * C, Lc = min(C, a.T - c0), r = t >> 2, qq = t & 3;
    if (r < Lc) {
      const float *src = a.dout + (((size_t)b * a.T + c0 + r) * H + h) * D + 32 * qq;
      uint8_t *dst = sm + R_STG + r * 512 + qq * 128;
#pragma unroll
      for (int e = 0; e < 8; ++e) cp_async16(dst + 16 * e, src + 4 * e);
    }
    cp_async_commit();
  };
  uint32_t ph_mma = 0;
  bool ok = true;
  if (t == 0) load_tiles(n - 1, 0);
  load_dout(n - 1);
#pragma unroll 1
  for (int it = 0; it < n && ok; ++it) {
    const int ci = n - 1 - it, st = it & 1;
    const int t0 = ci * C, L = min(C, a.T - t0);
    uint8_t *kqp = sm + R_KQ + st * 4 * kTile, *ttp = sm + R_TT + st * kTile;
    const uint32_t kq = smem_u32(kqp), tt = smem_u32(ttp);
    // the next chunk's K, Q, T into the other stage: every MMA and every
    // thread's access of the chunk before this one, which used it, is done
    if (ci >= 1 && t == 0) load_tiles(ci - 1, st ^ 1);
    if (warp == 0) {
      const size_t tok = ((size_t)b * a.T + t0 + lane) * H + h;
      float x0 = lane < L ? a.g[tok] : 0.f;
      float x1 = lane + 32 < L ? a.g[tok + (size_t)32 * H] : 0.f;
      const float gl = cumsum64(x0, x1, lane);
      gcv[lane] = x0;
      gcv[lane + 32] = x1;
      bv[lane] = __expf(x0);
      bv[lane + 32] = __expf(x1);
      kbv[lane] = __expf(gl - x0);
      kbv[lane + 32] = __expf(gl - x1);
    }
    {  // dO rows (this thread's own asynchronous copies) -> bf16 tile: row t / 4,
       // channels 32 (t % 4) .. + 31 (tile (t % 4) / 2, 16-byte chunks 4 ((t % 4) % 2) ..)
      const int r = t >> 2, qq = t & 3, hh = qq >> 1;
      cp_async_wait_all();
      uint8_t *tile = sm + R_DO + hh * kTile;
      const float4 *src = reinterpret_cast<const float4 *>(sm + R_STG + r * 512 + hh * 256);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const int ch = 4 * (qq & 1) + ((c4 + r) & 3);  // rotated: reads spread over the banks
        const float4 v0 = r < L ? src[2 * ch] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 v1 = r < L ? src[2 * ch + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<uint4 *>(tile + sw128_off(r, 8 * ch)) =
            make_uint4(pack_bf16(v0.x, v0.y), pack_bf16(v0.z, v0.w), pack_bf16(v1.x, v1.y),
                       pack_bf16(v1.z, v1.w));
      }
    }
    fence_proxy_async_smem();  // the dO tiles -> the bulk copy's reads
    __syncthreads();           // gate vectors written
    if (t == 0)  // the bf16 dO tiles of this chunk, for the gradient pass
      bulk_store(a.stash_do + ((size_t)bh * n + ci) * 2 * kTile, sm + R_DO, 2 * kTile);
    if (ci >= 1) load_dout(ci - 1);
    {  // dS1 -> its bf16 copy (TMEM) and the stash; dS <- e^{gl} dS1
      const float bl = bv[63];
      uint4 *dst = reinterpret_cast<uint4 *>(a.stash_ds + (((size_t)bh * n + ci) * D + i) * D);
#pragma unroll 1
      for (int q = hs; q < 4; q += 2) {
        float x[32];
        tmem_ld32(lb + TR_DS + 32 * q, x);
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        tmem_st16u(lb + TR_DSB + 16 * q, u);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[4 * q + e] = make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= bl;
        tmem_st32(lb + TR_DS + 32 * q, x);
      }
      tmem_wait_st();
    }
    ok = wait_all_threads(bar_ld + st, (it >> 1) & 1, ok);
    if (!ok) break;
    // ---- D1 = [K; Q] K^T (rows 64-127: Q K^T for P)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 2 * kTile + (kk & 3) * 32;
        mma_bf16_ss(tm + TR_D1, sdesc_sw128(kq + off, 16, 1024), sdesc_sw128(kq + off, 16, 1024),
                    ID_D1, kk > 0);
      }
      mma_commit(bar_mma);
    }
    {  // meanwhile: K-bar = K e^{gl - gc} (new tiles); T~ = T Diag(e^{gc}) in place
      const int r = t >> 2, qq = t & 3, hh = qq >> 1;
      const float f = kbv[r];
      const uint8_t *src = kqp + 2 * hh * kTile;
      uint8_t *dst = sm + R_KB + hh * kTile;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint32_t off = sw128_off(r, 8 * (4 * (qq & 1) + c4));
        *reinterpret_cast<uint4 *>(dst + off) = *reinterpret_cast<const uint4 *>(src + off);
        scale_chunk(dst + off, f);
      }
      // T~: row s = t / 4, columns 16 (t % 4) .. + 15 scaled by e^{gc_col}
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col = 16 * qq + 8 * ch;
        uint8_t *p = ttp + sw128_off(r, col);
        uint4 v = *reinterpret_cast<uint4 *>(p);
        uint32_t *w = &v.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = unpack_bf16(w[e]);
          w[e] = pack_bf16(x.x * bv[col + 2 * e], x.y * bv[col + 2 * e + 1]);
        }
        *reinterpret_cast<uint4 *>(p) = v;
      }
    }
    ok = wait_all_threads(bar_mma, ph_mma, ok);
    ph_mma ^= 1;
    if (!ok) break;
    tc_fence_after();
    // ---- P = tril(Q K^T e^{gc_r - gc_s}) (TMEM lanes 64-127); Q~ = Q Diag(e^{gc}) in place
    if (lq >= 2) {  // TMEM lanes 64-127 (rows r of Q K^T), columns 32 hs ..
      const int r = i - 64;
      float x[32];
      {
        const int hp = hs;
        tmem_ld32(lb + TR_D1 + 32 * hp, x);
        const float gr = gcv[r];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int s = 32 * hp + e;
          x[e] = (s <= r && r < L) ? x[e] * __expf(gr - gcv[s]) : 0.f;
        }
        st_row32(sm + R_P, r, hp, x);
      }
    }
    {
      const int r = t >> 2, qq = t & 3, hh = qq >> 1;
      uint8_t *qt = kqp + (2 * hh + 1) * kTile;
      const float f = bv[r];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) scale_chunk(qt + sw128_off(r, 8 * (4 * (qq & 1) + c4)), f);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- dV'^T = dO^T P + dS1 K-bar^T
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TR_DVP, sdesc_sw128(dq + kk * 2048, kTile, 1024),
                    sdesc_sw128(pp + kk * 2048, kTile, 1024), ID_DOP, kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tm + TR_DVP, tm + TR_DSB + 8 * kk,
               sdesc_sw128(kb + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024), ID_KB, 1);
      mma_commit(bar_mma);
    }
    ok = wait_all_threads(bar_mma, ph_mma, ok);
    ph_mma ^= 1;
    if (!ok) break;
    tc_fence_after();
    {  // dV'^T -> the stash and its bf16 copy in place: columns 32 hs .., all
       // reads before the writes
      float x0[32];
      tmem_ld32(lb + TR_DVP + 32 * hs, x0);
      uint32_t u[16];
      uint4 *dst = reinterpret_cast<uint4 *>(a.stash_dv + (((size_t)bh * n + ci) * D + i) * C);
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x0[2 * e], x0[2 * e + 1]);
      __syncthreads();
      tmem_st16u(lb + TR_DVP + 16 * hs, u);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        dst[4 * hs + e] = make_uint4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3]);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- Zc = dV'^T T~ ;  dS += dO^T Q~
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tm + TR_ZC, tm + TR_DVP + 8 * kk, sdesc_sw128(tt + kk * 2048, kTile, 1024), ID_ZC,
               kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TR_DS, sdesc_sw128(dq + kk * 2048, kTile, 1024),
                    sdesc_sw128(kq + kTile + kk * 2048, 2 * kTile, 1024), ID_DOQ, 1);
      mma_commit(bar_mma);
    }
    ok = wait_all_threads(bar_mma, ph_mma, ok);
    ph_mma ^= 1;
    if (!ok) break;
    tc_fence_after();
    {  // -Zc -> bf16 in place: columns 32 hs .., all reads before the writes
      float x0[32];
      tmem_ld32(lb + TR_ZC + 32 * hs, x0);
      uint32_t u[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = pack_bf16(-x0[2 * e], -x0[2 * e + 1]);
      __syncthreads();
      tmem_st16u(lb + TR_ZC + 16 * hs, u);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- dS += (-Zc) K
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tm + TR_DS, tm + TR_ZC + 8 * kk, sdesc_sw128(kq + kk * 2048, 2 * kTile, 1024),
               ID_ZK, 1);
      mma_commit(bar_mma);
      bulk_wait_read();  // the dO tiles are rewritten by the next chunk (after this barrier)
    }
    ok = wait_all_threads(bar_mma, ph_mma, ok);
    ph_mma ^= 1;
    tc_fence_after();
  }
  if (ok && a.dS0) {
#pragma unroll 1
    for (int q = hs; q < 4; q += 2) {
      float x[32];
      tmem_ld32(lb + TR_DS + 32 * q, x);
      float4 *dst = reinterpret_cast<float4 *>(a.dS0 + ((size_t)bh * D + i) * D + 32 * q);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
    }
  }
  cp_async_wait_all();
  if (t == 0) bulk_wait_all();
  if (!ok && t == 0) {  // a load still in flight lands before the CTA ends
    atomicOr(a.status, kStatusTimeout);
    if (ld_n0) mbar_wait_bounded(bar_ld, (uint32_t)(ld_n0 - 1) & 1u, kWaitNs);
    if (ld_n1) mbar_wait_bounded(bar_ld + 1, (uint32_t)(ld_n1 - 1) & 1u, kWaitNs);
  }
  if (t == 0) {  // every issued MMA has completed before TMEM is released
    mma_commit(bar_mma);
    mbar_wait_bounded(bar_mma, ph_mma, kWaitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

}  // namespace
}  // namespace gdr

namespace gdr {
namespace {

// ====================================================================== gradients
struct GradArgs {
  const float *g, *beta;  // [B, T, H]
  const uint8_t *stash_do;  // [B H n][16 KB]: the state pass's bf16 dO tiles
  float *dq, *dk, *dv;    // [B, T, H, D] fp32 (written)
  float *dg, *dbeta;      // [B, T, H] fp32 (written)
  int B, T, H, n;
};

// Shared memory: 8 KB tiles (128-byte swizzle), then vectors and barriers.
//   KQ [K_h0|Q_h0|K_h1|Q_h1], V [V_h0|V_h1] and dW^T [2] (contiguous: 32 KB
//   for the final reduction once both are dead), X0 [4], dS1 [4] (as
//   [rows 0-63: cols 0-63 | 64-127, rows 64-127: ...]), V'^T [2], dV'^T [2],
//   T, dO [2], Y, dY^T, dPs, dMs.
constexpr uint32_t G_KQ = 0, G_V = 4 * kTile, G_DWT = 6 * kTile, G_X = 8 * kTile,
                   G_DS = 12 * kTile, G_VP = 16 * kTile, G_DV = 18 * kTile, G_T = 20 * kTile,
                   G_DO = 21 * kTile, G_Y = 23 * kTile, G_DYT = 24 * kTile, G_DPS = 25 * kTile,
                   G_DMS = 26 * kTile, G_VEC = 27 * kTile, G_BAR = G_VEC + 4096,
                   G_MISC = G_BAR + 64, G_END = G_MISC + 64;
constexpr size_t kGradSmem = G_END + 1024;
static_assert(kGradSmem <= 232448, "shared memory budget");
// TMEM accumulator slots (64 columns each)
constexpr uint32_t TG0 = 0, TG1 = 64, TG2 = 128, TG3 = 192, TG4 = 256, TG5 = 320, TG6 = 384,
                   TG7 = 448;

__global__ void __launch_bounds__(kGradThreads, 1)
    gdr_bwd_grad_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmDS,
                        const __grid_constant__ CUtensorMap tmVP,
                        const __grid_constant__ CUtensorMap tmDV,
                        const __grid_constant__ CUtensorMap tmT, GradArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~uintptr_t(1023));
  // 8 warps: warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31 and
  // split each per-lane phase's columns between them (hs)
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, lq = warp & 3, hs = warp >> 2;
  const int ci = blockIdx.x % a.n, bh = blockIdx.x / a.n, b = bh / a.H, h = bh % a.H;
  const int H = a.H, t0 = ci * C, L = min(C, a.T - t0);
  const int chunk = bh * a.n + ci;
  uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + G_BAR), *bar_mma = bar_ld + 1;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + G_MISC);
  float *gcv = reinterpret_cast<float *>(sm + G_VEC);  // [64] cumulative log decay
  float *bv = gcv + 64;                                 // e^{gc}
  float *kbv = gcv + 128;                               // e^{gl - gc}
  float *betav = gcv + 192;                             // beta
  float *rbeta = gcv + 256;                             // 1 / beta (0 where beta = 0)
  float *dbeta1 = gcv + 320;                            // [2][64] column sums of dT . Y
  float *dbeta2s = gcv + 448;                           // [2][64] sums of dA M
  float *red = gcv + 576;                               // [8] block reduction
  float *scan = gcv + 640;                              // [64] scan scratch
  float *psum = gcv + 704;                              // [4][64] gate partial sums
  if (t == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_mma, 1);
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
  const int i = lq * 32 + lane;  // this thread's TMEM lane
  const uint32_t s_kq = smem_u32(sm + G_KQ), s_v = smem_u32(sm + G_V), s_x = smem_u32(sm + G_X);
  const uint32_t s_ds = smem_u32(sm + G_DS), s_vp = smem_u32(sm + G_VP);
  const uint32_t s_dv = smem_u32(sm + G_DV), s_t = smem_u32(sm + G_T), s_do = smem_u32(sm + G_DO);
  const uint32_t s_y = smem_u32(sm + G_Y), s_dyt = smem_u32(sm + G_DYT);
  const uint32_t s_dps = smem_u32(sm + G_DPS), s_dms = smem_u32(sm + G_DMS);
  const uint32_t s_dwt = smem_u32(sm + G_DWT);
  // operands with M = 128 whose rows 64-127 are not needed read the next 8 KB
  // (any data; those accumulator rows are never used)
  uint32_t ph = 0;
  bool ok = true;
  auto mma_wait = [&]() {
    if (t == 0) mma_commit(bar_mma);
    ok = wait_all_threads(bar_mma, ph, ok);
    ph ^= 1;
    tc_fence_after();
  };
  auto sync_for_mma = [&]() {  // generic smem / TMEM writes -> the next MMA
    fence_proxy_async_smem();
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // ---- loads
  if (t == 0) {
    mbar_arrive_expect_tx(bar_ld, 21 * kTile);  // K, Q, V, X0, dS1, V'^T, dV'^T, T, dO
    tma_load_4d(sm + G_KQ + 0 * kTile, &tmK, bar_ld, 0, h, t0, b);
    tma_load_4d(sm + G_KQ + 1 * kTile, &tmQ, bar_ld, 0, h, t0, b);
    tma_load_4d(sm + G_KQ + 2 * kTile, &tmK, bar_ld, 64, h, t0, b);
    tma_load_4d(sm + G_KQ + 3 * kTile, &tmQ, bar_ld, 64, h, t0, b);
    tma_load_4d(sm + G_V + 0 * kTile, &tmV, bar_ld, 0, h, t0, b);
    tma_load_4d(sm + G_V + 1 * kTile, &tmV, bar_ld, 64, h, t0, b);
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2)
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        tma_load_3d(sm + G_X + (2 * r2 + c2) * kTile, &tmX, bar_ld, 64 * c2, 64 * r2, chunk);
        tma_load_3d(sm + G_DS + (2 * r2 + c2) * kTile, &tmDS, bar_ld, 64 * c2, 64 * r2, chunk);
      }
    tma_load_3d(sm + G_VP + 0 * kTile, &tmVP, bar_ld, 0, 0, chunk);
    tma_load_3d(sm + G_VP + 1 * kTile, &tmVP, bar_ld, 0, 64, chunk);
    tma_load_3d(sm + G_DV + 0 * kTile, &tmDV, bar_ld, 0, 0, chunk);
    tma_load_3d(sm + G_DV + 1 * kTile, &tmDV, bar_ld, 0, 64, chunk);
    tma_load_3d(sm + G_T, &tmT, bar_ld, 0, 0, chunk);
    // dO (bf16, already in the tiles' swizzled layout, from the state pass)
    bulk_load(sm + G_DO, a.stash_do + (size_t)chunk * 2 * kTile, 2 * kTile, bar_ld);
  }
  if (warp == 0) {  // gates
    const size_t tok = ((size_t)b * a.T + t0 + lane) * H + h;
    float x0 = lane < L ? a.g[tok] : 0.f;
    float x1 = lane + 32 < L ? a.g[tok + (size_t)32 * H] : 0.f;
    const float gl = cumsum64(x0, x1, lane);
    gcv[lane] = x0;
    gcv[lane + 32] = x1;
    bv[lane] = __expf(x0);
    bv[lane + 32] = __expf(x1);
    kbv[lane] = __expf(gl - x0);
    kbv[lane + 32] = __expf(gl - x1);
    const float b0 = lane < L ? a.beta[tok] : 0.f;
    const float b1 = lane + 32 < L ? a.beta[tok + (size_t)32 * H] : 0.f;
    betav[lane] = b0;
    betav[lane + 32] = b1;
    rbeta[lane] = b0 > 0.f ? 1.f / b0 : 0.f;
    rbeta[lane + 32] = b1 > 0.f ? 1.f / b1 : 0.f;
  }
  ok = wait_all_threads(bar_ld, 0, ok);
  sync_for_mma();

  const size_t row0 = ((size_t)b * a.T + t0) * H + h;  // token index of row 0
  if (ok) {
    // ---- G1: dV^T = dV'^T T  [i][r];  G3a: dT^T_1 = V dV'^T [s][r];
    //      G2: dW^T = -X0 dV'^T [j][r];  G7: KK = K K^T [s][p]
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG0, sdesc_sw128(s_dv + kk * 32, 16, 1024),
                    sdesc_sw128(s_t + kk * 2048, kTile, 1024), idesc_bf16(128, 64, 0, 1), kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG1, sdesc_sw128(s_v + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(s_dv + (kk >> 2) * kTile + (kk & 3) * 2048, kTile, 1024),
                    idesc_bf16(128, 64, 0, 1), kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG2, sdesc_sw128(s_x + (kk >> 2) * 2 * kTile + (kk & 3) * 2048, kTile, 1024),
                    sdesc_sw128(s_dv + (kk >> 2) * kTile + (kk & 3) * 2048, kTile, 1024),
                    idesc_bf16(128, 64, 1, 1, /*neg_a=*/1), kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 2 * kTile + (kk & 3) * 32;
        mma_bf16_ss(tm + TG4, sdesc_sw128(s_kq + off, 16, 1024), sdesc_sw128(s_kq + off, 16, 1024),
                    idesc_bf16(128, 64, 0, 0), kk > 0);
      }
    }
    mma_wait();
  }
  if (ok) {
    // dv (lanes = value channels); dW^T -> bf16 (TMEM in place, and the smem
    // tile [j][r]); Y = T Diag(1 / beta) (rows r < 64)
    {  // tokens 32 hs .. 32 hs + 31
      float x0[32];
      tmem_ld32(lb + TG0 + 32 * hs, x0);
      float *dst = a.dv + row0 * D + i;
      const size_t rs = (size_t)H * D;
#pragma unroll
      for (int r = 0; r < 32; ++r)
        if (32 * hs + r < L) dst[(32 * hs + r) * rs] = x0[r];
    }
    {  // columns 32 hs ..: all reads of the fp32 dW^T before its bf16 copy overwrites it
      float x0[32];
      tmem_ld32(lb + TG2 + 32 * hs, x0);
      uint32_t u[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x0[2 * e], x0[2 * e + 1]);
      __syncthreads();
      tmem_st16u(lb + TG2 + 16 * hs, u);
      st_row32(sm + G_DWT + (i >> 6) * kTile, i & 63, hs, x0);
    }
    if (t < 128) {  // row r of Y from row r of T, half t / 64 of the columns
      const int r = t & 63;
      float y[32];
      {
        const int hp = t >> 6;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4 *>(sm + G_T + sw128_off(r, 32 * hp + 8 * ch));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int s = 32 * hp + 8 * ch + 2 * e;
            const float2 x = unpack_bf16(w[e]);
            const float b0 = betav[s], b1 = betav[s + 1];
            y[8 * ch + 2 * e] = b0 > 0.f ? x.x * rbeta[s] : (r == s ? 1.f : 0.f);
            y[8 * ch + 2 * e + 1] = b1 > 0.f ? x.y * rbeta[s + 1] : (r == s + 1 ? 1.f : 0.f);
          }
        }
        st_row32(sm + G_Y, r, hp, y);
      }
    }
    sync_for_mma();
    // ---- G3b: dT^T_2 = K dW^T [s][r]
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG3, sdesc_sw128(s_kq + (kk >> 2) * 2 * kTile + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(s_dwt + (kk >> 2) * kTile + (kk & 3) * 2048, kTile, 1024),
                    idesc_bf16(128, 64, 0, 1), kk > 0);
    }
    mma_wait();
  }
  if (ok) {
    // dT^T [s][r] = dT^T_1 + e^{gc_s} dT^T_2 (rows s < 64): dbeta_s (part 1) =
    // sum_r dT[r][s] Y[r][s]; dY^T [s][r] = beta_s dT^T[s][r]
    if (lq < 2) {  // rows s = lanes 0-63, columns 32 hs ..
      const int s = i;
      float x[32], y2[32];
      float acc = 0.f;
      const float bs = bv[s], bes = betav[s];
      {
        const int hp = hs;
        tmem_ld32(lb + TG1 + 32 * hp, x);
        tmem_ld32(lb + TG3 + 32 * hp, y2);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int r = 32 * hp + e;
          x[e] += bs * y2[e];
          const uint16_t yb = *reinterpret_cast<const uint16_t *>(sm + G_Y + sw128_off(r, s));
          acc += x[e] * __uint_as_float((uint32_t)yb << 16);
          x[e] *= bes;
        }
        st_row32(sm + G_DYT, s, hp, x);
      }
      dbeta1[64 * hs + s] = acc;
    }
    sync_for_mma();
    // ---- G5: E = Y^T dY [s][q]
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG1, sdesc_sw128(s_y + kk * 2048, kTile, 1024),
                    sdesc_sw128(s_dyt + kk * 32, 16, 1024), idesc_bf16(128, 64, 1, 0), kk > 0);
    }
    mma_wait();
  }
  if (ok) {
    {  // E -> bf16 in place (A of G6): columns 32 hs .., all reads before the writes
      float x0[32];
      tmem_ld32(lb + TG1 + 32 * hs, x0);
      uint32_t u[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) u[e] = pack_bf16(x0[2 * e], x0[2 * e + 1]);
      __syncthreads();
      tmem_st16u(lb + TG1 + 16 * hs, u);
    }
    sync_for_mma();
    // ---- G6: F = E Y^T [s][p];  G8a: dP = dO V'^T [r][s]
    if (t == 0) {
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tm + TG3, tm + TG1 + 8 * kk, sdesc_sw128(s_y + kk * 32, 16, 1024),
               idesc_bf16(128, 64, 0, 0), kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG5, sdesc_sw128(s_do + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(s_vp + (kk >> 2) * kTile + (kk & 3) * 2048, kTile, 1024),
                    idesc_bf16(128, 64, 0, 1), kk > 0);
    }
    mma_wait();
  }
  float dbeta2 = 0.f;
  if (ok) {
    // rows s < 64: dA = strict_tril(-F); dbeta_s (part 2) = sum_p dA M, M =
    // KK e^{gc_s - gc_p}; dMs[s][p] = beta_s dA[s][p] e^{gc_s - gc_p};
    // dPs[r][s] = tril(dP)[r][s] e^{gc_r - gc_s}
    if (lq < 2) {  // rows r = lanes 0-63, columns 32 hs ..
      const int r = i;
      const float gr = gcv[r], br = betav[r];
      float f[32], kk2[32], p[32];
      {
        const int hp = hs;
        tmem_ld32(lb + TG3 + 32 * hp, f);
        tmem_ld32(lb + TG4 + 32 * hp, kk2);
        tmem_ld32(lb + TG5 + 32 * hp, p);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int s = 32 * hp + e;
          const float dec = s <= r ? __expf(gr - gcv[s]) : 0.f;
          const float da = s < r ? -f[e] : 0.f;
          dbeta2 += da * kk2[e] * dec;
          f[e] = br * da * dec;
          p[e] = (r < L) ? p[e] * dec : 0.f;
        }
        st_row32(sm + G_DMS, r, hp, f);
        st_row32(sm + G_DPS, r, hp, p);
      }
      dbeta2s[64 * hs + r] = dbeta2;
    }
    // dO -> dO~ = Diag(e^{gc}) dO; V'^T columns scaled by e^{gl - gc};
    // T -> T~ = T Diag(e^{gc}) (all in place; their unscaled uses are done)
    {
      // dO~: 64 rows x 2 tiles x 8 chunks, four 16-byte chunks per thread
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int id = t + 256 * k, r = id >> 4, hh = (id >> 3) & 1, ch = id & 7;
        scale_chunk(sm + G_DO + hh * kTile + sw128_off(r, 8 * ch), bv[r]);
      }
      // V'^T: rows i (128) x 8 chunks of columns r, four per thread
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int id = t + 256 * k, row = id >> 3, ch = id & 7;
        uint8_t *p = sm + G_VP + (row >> 6) * kTile + sw128_off(row & 63, 8 * ch);
        uint4 v = *reinterpret_cast<uint4 *>(p);
        uint32_t *w = &v.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = unpack_bf16(w[e]);
          w[e] = pack_bf16(x.x * kbv[8 * ch + 2 * e], x.y * kbv[8 * ch + 2 * e + 1]);
        }
        *reinterpret_cast<uint4 *>(p) = v;
      }
      // T: 64 rows x 8 chunks, columns scaled by e^{gc_col}, two per thread
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int id = t + 256 * k, row = id >> 3, ch = id & 7;
        uint8_t *p = sm + G_T + sw128_off(row, 8 * ch);
        uint4 v = *reinterpret_cast<uint4 *>(p);
        uint32_t *w = &v.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = unpack_bf16(w[e]);
          w[e] = pack_bf16(x.x * bv[8 * ch + 2 * e], x.y * bv[8 * ch + 2 * e + 1]);
        }
        *reinterpret_cast<uint4 *>(p) = v;
      }
    }
    sync_for_mma();
    // ---- G8: AccQ [j][r] = X0 dO~^T + K^T dPs^T;  G9: AccH [j][s] = Q^T dPs + K^T dMs;
    //      G10: AccT [j][r] = dW^T T~ + K^T dMs^T;  G11: AccB [j][r] = dS1^T (V'^T scaled)
    if (t == 0) {
      const uint32_t ID_QX = idesc_bf16(128, 64, 1, 0);   // A MN-major, B K-major
      const uint32_t ID_MNMN = idesc_bf16(128, 64, 1, 1);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG6, sdesc_sw128(s_x + (kk >> 2) * 2 * kTile + (kk & 3) * 2048, kTile, 1024),
                    sdesc_sw128(s_do + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024), ID_QX, kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG6, sdesc_sw128(s_kq + kk * 2048, 2 * kTile, 1024),
                    sdesc_sw128(s_dps + kk * 32, 16, 1024), ID_QX, 1);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG7, sdesc_sw128(s_kq + kTile + kk * 2048, 2 * kTile, 1024),
                    sdesc_sw128(s_dps + kk * 2048, kTile, 1024), ID_MNMN, kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG7, sdesc_sw128(s_kq + kk * 2048, 2 * kTile, 1024),
                    sdesc_sw128(s_dms + kk * 2048, kTile, 1024), ID_MNMN, 1);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(tm + TG1, tm + TG2 + 8 * kk, sdesc_sw128(s_t + kk * 2048, kTile, 1024),
               idesc_bf16(128, 64, 0, 1), kk > 0);
#pragma unroll 1
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tm + TG1, sdesc_sw128(s_kq + kk * 2048, 2 * kTile, 1024),
                    sdesc_sw128(s_dms + kk * 32, 16, 1024), ID_QX, 1);
#pragma unroll 1
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tm + TG3, sdesc_sw128(s_ds + (kk >> 2) * 2 * kTile + (kk & 3) * 2048, kTile, 1024),
                    sdesc_sw128(s_vp + (kk >> 2) * kTile + (kk & 3) * 2048, kTile, 1024), ID_MNMN,
                    kk > 0);
    }
    mma_wait();
  }
  if (ok) {
    // lanes = key channels j: dq = AccQ, dk = AccT + AccH + AccB; gate
    // partials p[j][r] = (AccT - AccH - AccB) K[r][j] + AccQ Q[r][j] into the
    // (now dead) V and dW^T tiles, fp32 [128][64], entry (j, r) at column
    // r ^ (j % 32) (writes by lanes j and reads by lanes r hit distinct banks)
    const int j = lq * 32 + lane;
    float *part = reinterpret_cast<float *>(sm + G_V);
    const uint8_t *kt = sm + G_KQ + 2 * (j >> 6) * kTile, *qt = kt + kTile;
    float dbl = 0.f;  // sum over r of AccB K
    {  // tokens 32 hs .. 32 hs + 31
      const int hp = hs;
      float aq[32], at[32], ah[32], ab[32];
      tmem_ld32(lb + TG6 + 32 * hp, aq);
      tmem_ld32(lb + TG1 + 32 * hp, at);
      tmem_ld32(lb + TG7 + 32 * hp, ah);
      tmem_ld32(lb + TG3 + 32 * hp, ab);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int r = 32 * hp + e;
        const float kv = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(
                                             kt + sw128_off(r, j & 63)) << 16);
        const float qv = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(
                                             qt + sw128_off(r, j & 63)) << 16);
        part[j * 64 + (r ^ (j & 31))] = (at[e] - ah[e] - ab[e]) * kv + aq[e] * qv;
        dbl += ab[e] * kv;
        if (r < L) {
          const size_t o = (row0 + (size_t)r * H) * D + j;
          a.dq[o] = aq[e];
          a.dk[o] = at[e] + ah[e] + ab[e];
        }
      }
    }
    // + e^{gl} sum_ij dS1 X0 (row i = j of this thread)
    {
      const uint8_t *dsr = sm + G_DS + 2 * (j >> 6) * kTile, *xr = sm + G_X + 2 * (j >> 6) * kTile;
      float acc = 0.f;
      {
        const int hc = hs;  // columns 64 hs .. 64 hs + 63 of the row
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t off = hc * kTile + sw128_off(j & 63, 8 * ch);
          const uint4 u = *reinterpret_cast<const uint4 *>(dsr + off);
          const uint4 w = *reinterpret_cast<const uint4 *>(xr + off);
          const uint32_t uu[4] = {u.x, u.y, u.z, u.w}, ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 p = unpack_bf16(uu[e]), q = unpack_bf16(ww[e]);
            acc += p.x * q.x + p.y * q.y;
          }
        }
      }
      dbl += bv[63] * acc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dbl += __shfl_xor_sync(0xffffffffu, dbl, off);
    if (lane == 0) red[warp] = dbl;
    __syncthreads();
    {  // partial sums of the gate partials over 32 key channels each
      const int r = t & 63, qj = t >> 6;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll 2
      for (int jj = 32 * qj; jj < 32 * qj + 32; jj += 4) {
        s0 += part[(jj + 0) * 64 + (r ^ ((jj + 0) & 31))];
        s1 += part[(jj + 1) * 64 + (r ^ ((jj + 1) & 31))];
        s2 += part[(jj + 2) * 64 + (r ^ ((jj + 2) & 31))];
        s3 += part[(jj + 3) * 64 + (r ^ ((jj + 3) & 31))];
      }
      psum[64 * qj + r] = (s0 + s1) + (s2 + s3);
    }
    __syncthreads();
    if (t < 64) {  // dgc_r, then the reverse cumsum within the chunk; dbeta
      const int r = t;
      float s = (psum[r] + psum[64 + r]) + (psum[128 + r] + psum[192 + r]);
      if (r == 63)
        s += ((red[0] + red[1]) + (red[2] + red[3])) + ((red[4] + red[5]) + (red[6] + red[7]));
      // reverse inclusive scan over r within two warps (rows 0-31, 32-63)
      float x = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, x, off);
        if (lane + off < 32) x += y;
      }
      scan[r] = x;
      const float db = (dbeta2s[r] + dbeta2s[64 + r]) + (dbeta1[r] + dbeta1[64 + r]);
      if (r < L) a.dbeta[row0 + (size_t)r * H] = db;
    }
    __syncthreads();
    if (t < 64) {
      const int r = t;
      float x = scan[r];
      if (r < 32) x += scan[32];  // rows 32-63's total
      if (r < L) a.dg[row0 + (size_t)r * H] = x;
    }
  }
  if (t == 0) {  // every issued MMA has completed before TMEM is released
    mma_commit(bar_mma);
    mbar_wait_bounded(bar_mma, ph, kWaitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, 512);
}

}  // namespace
}  // namespace gdr

namespace gdr {

// Per-chunk stash of the tensor-core backward, bytes: X0 [128][128], V'^T
// [128][64], T [64][64], dS1 [128][128], dV'^T [128][64], dO [64][128], all
// bf16 (dO as the two 128-byte-swizzled tiles the state pass converted).
constexpr size_t kStashX = (size_t)D * D * 2, kStashV = (size_t)D * C * 2,
                 kStashT = (size_t)C * C * 2, kStashO = (size_t)C * D * 2;
constexpr size_t kStashPerChunk = 2 * kStashX + 2 * kStashV + kStashT + kStashO;

bool bwd_tc_supports(int bf16, int per_channel, int d) {
  return bf16 && !per_channel && d == D;
}

size_t bwd_tc_ws_bytes(int B, int T, int H) {
  if (B <= 0 || H <= 0 || T <= 0) return 0;
  return (size_t)B * H * ((T + C - 1) / C) * kStashPerChunk;
}

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *S0, const float *dout,
                          const float *dST, float *dq, float *dk, float *dv, float *dg,
                          float *dbeta, float *dS0, int B, int T, int H, void *ws,
                          unsigned int *status, cudaStream_t stream) {
  const long long n = (T + C - 1) / C, nch = (long long)B * H * n;
  if (nch <= 0) return cudaSuccess;
  if (nch > 0x7fffffffLL) return cudaErrorInvalidValue;
  uint8_t *w = static_cast<uint8_t *>(ws);
  __nv_bfloat16 *sx = reinterpret_cast<__nv_bfloat16 *>(w);
  __nv_bfloat16 *sv = reinterpret_cast<__nv_bfloat16 *>(w + nch * kStashX);
  __nv_bfloat16 *st = reinterpret_cast<__nv_bfloat16 *>(w + nch * (kStashX + kStashV));
  __nv_bfloat16 *sds = reinterpret_cast<__nv_bfloat16 *>(w + nch * (kStashX + kStashV + kStashT));
  __nv_bfloat16 *sdv = reinterpret_cast<__nv_bfloat16 *>(w + nch * (2 * kStashX + kStashV + kStashT));
  uint8_t *sdo = w + nch * (2 * kStashX + 2 * kStashV + kStashT);
  // 1. the forward again, stashing X0, V'^T and T per chunk (no o)
  ChunkArgs fa{};
  fa.q = q; fa.k = k; fa.v = v; fa.g = g; fa.beta = beta; fa.S0 = S0;
  fa.o = nullptr; fa.S_T = nullptr;
  fa.B = B; fa.T = T; fa.H = H; fa.dk = D; fa.dv = D;
  fa.bf16 = 1; fa.per_channel = 0; fa.status = status; fa.skip_stage_chunk = -1;
  fa.write_o = 0;
  fa.stash_x = sx; fa.stash_v = sv; fa.stash_t = st;
  cudaError_t e = launch_chunk_tc(fa, stream);
  if (e != cudaSuccess) return e;
  // 2. the state gradient, chunks in reverse
  CUtensorMap mq, mk, mv, mt, mx, mds, mvp, mdv;
  if (!tc_map_bf16(&mq, q, B, T, H, D) || !tc_map_bf16(&mk, k, B, T, H, D) ||
      !tc_map_bf16(&mv, v, B, T, H, D) || !tc_map_stash(&mt, st, nch, C, C) ||
      !tc_map_stash(&mx, sx, nch, D, D) || !tc_map_stash(&mds, sds, nch, D, D) ||
      !tc_map_stash(&mvp, sv, nch, D, C) || !tc_map_stash(&mdv, sdv, nch, D, C))
    return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(gdr_bwd_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kStateSmem);
  if (e != cudaSuccess) return e;
  StateArgs ra{g, dout, dST, dS0, sds, sdv, sdo, B, T, H, (int)n, status};
  gdr_bwd_state_kernel<<<(unsigned)(B * H), kStateThreads, kStateSmem, stream>>>(mk, mq, mt, ra);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3. the token gradients, one CTA per chunk and head
  e = cudaFuncSetAttribute(gdr_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kGradSmem);
  if (e != cudaSuccess) return e;
  GradArgs ga{g, beta, sdo, dq, dk, dv, dg, dbeta, B, T, H, (int)n};
  gdr_bwd_grad_kernel<<<(unsigned)nch, kGradThreads, kGradSmem, stream>>>(mq, mk, mv, mx, mds, mvp,
                                                                      mdv, mt, ga);
  return cudaGetLastError();
}

}  // namespace gdr
