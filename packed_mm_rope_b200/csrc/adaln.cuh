// adaln.cuh -- per-row AdaLN modulation before the attention projections.
//
// "MiniMax H3 -- one transformer that denoises video and audio together",
// AdaLN passage: y = norm(x) * (1 + scale) + shift, with (scale, shift) taken
// per row from a table indexed by (noise level, modality):
// adaln_indices = timestep_indices * 3 + token_tags.  "Inside MiniMax H3",
// section 5: the table is small (unique timesteps x modalities) and its
// entries are gathered for each row.  norm is LayerNorm without its own affine
// parameters (biased variance, eps given by the caller).
//
// HBM-bound: each row is read once and written once (2 x hidden x 2 bytes).
// A group of four warps owns a row at a time and holds it in registers (at
// most 8 x 16 bytes per thread, hidden <= 8192), so the row is read from DRAM
// once and the two passes (statistics, then modulation) run on registers.
// Eight such groups per SM (two per CTA, four CTAs per SM) keep enough loads
// in flight to stream at HBM speed; the table entry (8 bytes per column) is
// served by L1/L2, since a handful of entries cover all rows.  There are no
// waits on other threads beyond one barrier per row within a group.
#pragma once

#include "common.cuh"

namespace h3 {

constexpr int ADALN_THREADS = 256;                 // two row groups of four warps
constexpr int ADALN_GROUP = 128;                   // threads per row
constexpr int ADALN_GROUPS = ADALN_THREADS / ADALN_GROUP;
constexpr int ADALN_WARPS_PER_GROUP = ADALN_GROUP / 32;
constexpr int ADALN_CHUNKS_PER_THREAD = 8;         // 16-byte chunks of the row per thread
constexpr int ADALN_MAX_HIDDEN = ADALN_GROUP * ADALN_CHUNKS_PER_THREAD * 8;   // 8192
constexpr int ADALN_CTAS_PER_SM = 4;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Group g of CTA b takes rows b * ADALN_GROUPS + g, then every
// (gridDim.x * ADALN_GROUPS)-th row.  Thread t of the group holds the row's
// 16-byte chunks t, t + 128, ...  Statistics: one pass, shifted by the row's
// first element to avoid cancellation (mean = K + S1/n, var = S2/n - (S1/n)^2
// with S1 = sum(x - K), S2 = sum((x - K)^2)); each warp reduces with shuffles
// and the four warp partials meet in shared memory behind one named barrier
// per row (double-buffered by row parity, so the next row's partials never
// overwrite ones still being read).  x and y may be the same rows (in place):
// a group has read its whole row before it writes any of it.
__global__ void __launch_bounds__(ADALN_THREADS, ADALN_CTAS_PER_SM) adaln_kernel(
    const uint4* x, uint4* y, const int32_t* __restrict__ ts_idx, const int32_t* __restrict__ tags,
    const float4* __restrict__ table, int n_entries, long long n_rows, int chunks, long long x_stride16,
    long long y_stride16, float eps, int err_slot) {
  __shared__ float2 partial[ADALN_GROUPS][2][ADALN_WARPS_PER_GROUP];   // (S1, S2) per warp
  const int g = threadIdx.x / ADALN_GROUP;
  const int t = threadIdx.x % ADALN_GROUP;
  const int wq = t >> 5, lane = threadIdx.x & 31;
  const float inv_c = 1.f / static_cast<float>(chunks * 8);
  int parity = 0;
  for (long long r = static_cast<long long>(blockIdx.x) * ADALN_GROUPS + g; r < n_rows;
       r += static_cast<long long>(gridDim.x) * ADALN_GROUPS, parity ^= 1) {
    const uint4* xr = x + r * x_stride16;
    uint4 u[ADALN_CHUNKS_PER_THREAD];
#pragma unroll
    for (int i = 0; i < ADALN_CHUNKS_PER_THREAD; ++i)
      u[i] = (t + ADALN_GROUP * i < chunks) ? __ldcs(xr + t + ADALN_GROUP * i) : make_uint4(0u, 0u, 0u, 0u);
    const float kf = __uint_as_float(*reinterpret_cast<const uint32_t*>(xr) << 16);   // element 0
    const float2 k2 = make_float2(-kf, -kf);
    float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < ADALN_CHUNKS_PER_THREAD; ++i) {
      if (t + ADALN_GROUP * i >= chunks) continue;
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 d = __fadd2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[m])), k2);
        s1 = __fadd2_rn(s1, d);
        s2 = __ffma2_rn(d, d, s2);
      }
    }
    const float w1 = warp_sum(s1.x + s1.y), w2 = warp_sum(s2.x + s2.y);
    if (lane == 0) partial[g][parity][wq] = make_float2(w1, w2);
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(ADALN_GROUP) : "memory");
    float a1 = 0.f, a2 = 0.f;
#pragma unroll
    for (int q = 0; q < ADALN_WARPS_PER_GROUP; ++q) {
      const float2 v = partial[g][parity][q];
      a1 += v.x;
      a2 += v.y;
    }
    const float m1 = a1 * inv_c;
    const float var = fmaxf(a2 * inv_c - m1 * m1, 0.f);
    const float mean = kf + m1;
    const float rstd = rsqrtf(var + eps);
    const long long e = static_cast<long long>(ts_idx[r]) * 3 + tags[r];
    const bool bad = e < 0 || e >= n_entries;
    if (bad && t == 0) raise_error(err_slot, DEVERR_INPUT);
    const float4* ent = table + (bad ? 0 : e) * 4LL * chunks;
    // y = x * a + b with a = rstd * (1 + scale), b = shift - mean * a
    const float2 rs2 = make_float2(rstd, rstd), nm2 = make_float2(-mean, -mean), one2 = make_float2(1.f, 1.f);
    uint4* yr = y + r * y_stride16;
#pragma unroll
    for (int i = 0; i < ADALN_CHUNKS_PER_THREAD; ++i) {
      const int c = t + ADALN_GROUP * i;
      if (c >= chunks) continue;
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
      const float4 s0 = __ldg(ent + 2 * c), s1v = __ldg(ent + 2 * c + 1);
      const float4 g0 = __ldg(ent + 2 * chunks + 2 * c), g1 = __ldg(ent + 2 * chunks + 2 * c + 1);
      const float2 sh[4] = {make_float2(s0.x, s0.y), make_float2(s0.z, s0.w), make_float2(s1v.x, s1v.y),
                            make_float2(s1v.z, s1v.w)};
      const float2 gs[4] = {make_float2(g0.x, g0.y), make_float2(g0.z, g0.w), make_float2(g1.x, g1.y),
                            make_float2(g1.z, g1.w)};
      uint32_t o[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 a = __fmul2_rn(rs2, __fadd2_rn(gs[m], one2));
        const float2 b = __ffma2_rn(nm2, a, sh[m]);
        const float2 v = __ffma2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[m])), a, b);
        o[m] = bad ? 0x7fc07fc0u : pack_bf16x2(v.x, v.y);
      }
      __stcs(yr + c, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

}  // namespace h3
