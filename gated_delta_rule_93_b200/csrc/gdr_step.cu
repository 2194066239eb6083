// One recurrent decode step of the gated delta rule, N independent states.
//
// Source: "Decoding Hybrid Linear Attention Architectures", section 6 (each
// decoded token costs one constant-size update of the state) and section 3
// item 6 (decay, then erase along k, then write).  Per state row i (value
// channel) with S' = S Diag(alpha):
//     p_i = S'_i . k,  r_i = S'_i . q,  u_i = beta (v_i - p_i)
//     S_i <- S'_i + u_i k^T,  o_i = S_i . q = r_i + u_i (k . q)
// so every row is read once and written once: the kernel is a single
// streaming pass over S (2 * d_k * d_v * 4 bytes per state), bound by HBM.
//
// Layout: one warp owns 8 consecutive rows of one (n, h); lane l holds the
// key channels [l*VEC, l*VEC + VEC) of each row (VEC = d_k / 32), loaded as
// one 4/8/16-byte vector, so a row is one fully coalesced 128..512-byte
// transaction.  A block is 4 warps = 32 rows; grid = N * H * d_v / 32.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kRowsPerWarp = 8;
constexpr int kWarps = 4;

template <int VEC>
struct VecT;
template <>
struct VecT<1> { using T = float; };
template <>
struct VecT<2> { using T = float2; };
template <>
struct VecT<4> { using T = float4; };

template <int VEC>
__device__ __forceinline__ void ld_vec(const float *p, float (&x)[VEC]) {
  if constexpr (VEC == 4) {
    float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else if constexpr (VEC == 2) {
    float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
    x[0] = t.x; x[1] = t.y;
  } else {
    x[0] = __ldcs(p);
  }
}

template <int VEC>
__device__ __forceinline__ void st_vec(float *p, const float (&x)[VEC]) {
  if constexpr (VEC == 4) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
  } else if constexpr (VEC == 2) {
    __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
  } else {
    __stcs(p, x[0]);
  }
}

// Sum 16 per-lane values over the warp with a halving butterfly: after the
// call lane l holds the full sum of value index
//   idx(l) = 8*bit4(l) + 4*bit3(l) + 2*bit2(l) + bit1(l)
// (lanes l and l^1 hold the same value).  16 shuffles instead of 80.
__device__ __forceinline__ float reduce16(float (&x)[16], int lane) {
  float y8[8], y4[4], y2[2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float send = hi ? x[i] : x[i + 8];
    const float keep = hi ? x[i + 8] : x[i];
    y8[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    const float send = hi ? y8[i] : y8[i + 4];
    const float keep = hi ? y8[i + 4] : y8[i];
    y4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    const float send = hi ? y4[i] : y4[i + 2];
    const float keep = hi ? y4[i + 2] : y4[i];
    y2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const bool hi = lane & 2;
  const float send = hi ? y2[0] : y2[1];
  const float keep = hi ? y2[1] : y2[0];
  float y = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  return y;
}

template <int DK, bool BF16, bool PERCH>
__global__ void __launch_bounds__(kWarps * 32) gdr_step_kernel(StepArgs a) {
  constexpr int VEC = DK / 32;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int blocks_per_state = a.dv / (kWarps * kRowsPerWarp);
  const size_t nh = blockIdx.x / blocks_per_state;
  const int row0 = (blockIdx.x % blocks_per_state) * (kWarps * kRowsPerWarp) +
                   warp * kRowsPerWarp;
  const int j0 = lane * VEC;

  // Key, query and gate for this (n, h).
  float kv[VEC], qv[VEC], al[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    kv[e] = load_in(a.k, nh * DK + j0 + e, BF16);
    qv[e] = load_in(a.q, nh * DK + j0 + e, BF16);
  }
  if constexpr (PERCH) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) al[e] = __expf(a.g[nh * DK + j0 + e]);
  } else {
    const float a0 = __expf(a.g[nh]);
#pragma unroll
    for (int e = 0; e < VEC; ++e) al[e] = a0;
  }
  const float beta = a.beta[nh];
  float kq = 0.f;
#pragma unroll
  for (int e = 0; e < VEC; ++e) kq += kv[e] * qv[e];
#pragma unroll
  for (int off = 16; off; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);

  float *Srow = a.S + (nh * a.dv + row0) * DK + j0;
  float s[kRowsPerWarp][VEC];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) ld_vec<VEC>(Srow + (size_t)r * DK, s[r]);

  // Lane r < 8 fetches v of row r.
  float vrow = 0.f;
  if (lane < kRowsPerWarp) vrow = load_in(a.v, nh * a.dv + row0 + lane, BF16);

  float part[16];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    float p = 0.f, rr = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      s[r][e] *= al[e];  // decay first
      p += s[r][e] * kv[e];
      rr += s[r][e] * qv[e];
    }
    part[r] = p;
    part[8 + r] = rr;
  }
  const float red = reduce16(part, lane);
  // Lane 2r holds p_r, lane 16 + 2r holds r_r.
  const int my_row = (lane >> 1) & 7;
  const float v_my = __shfl_sync(0xffffffffu, vrow, my_row);
  const float u_mine = beta * (v_my - red);  // meaningful on lanes < 16
  float u[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) u[r] = __shfl_sync(0xffffffffu, u_mine, 2 * r);
  if (lane >= 16 && !(lane & 1)) {
    const int r = my_row;
    store_out(a.o, nh * a.dv + row0 + r, red + u[r] * kq, BF16);
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) s[r][e] += u[r] * kv[e];
    st_vec<VEC>(Srow + (size_t)r * DK, s[r]);
  }
}

template <int DK>
cudaError_t launch_dk(const StepArgs &a, cudaStream_t stream) {
  const size_t blocks = (size_t)a.N * a.H * (a.dv / (kWarps * kRowsPerWarp));
  if (blocks > 0x7fffffffu) return cudaErrorInvalidValue;
  dim3 grid((unsigned)blocks), block(kWarps * 32);
  if (a.bf16) {
    if (a.per_channel)
      gdr_step_kernel<DK, true, true><<<grid, block, 0, stream>>>(a);
    else
      gdr_step_kernel<DK, true, false><<<grid, block, 0, stream>>>(a);
  } else {
    if (a.per_channel)
      gdr_step_kernel<DK, false, true><<<grid, block, 0, stream>>>(a);
    else
      gdr_step_kernel<DK, false, false><<<grid, block, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepArgs &a, cudaStream_t stream) {
  switch (a.dk) {
    case 32: return launch_dk<32>(a, stream);
    case 64: return launch_dk<64>(a, stream);
    case 128: return launch_dk<128>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gdr
