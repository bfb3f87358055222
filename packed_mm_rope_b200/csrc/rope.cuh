// rope.cuh -- fused three-axis MM-RoPE rotation of bf16 Q and K.
//
// "Inside MiniMax H3" section 4 and the model card's H3-Omni-Transformer
// section: Q and K are rotated by a (t, h, w) rotary embedding; the explainer
// page traces position_ids[:, 0] (t) into rope() and the rotation of Q and K,
// with inverse frequencies computed from rope_theta / rope_freq_dim.
//
// HBM-bound streaming kernel: one warp per packed row streams both tensors
// with 16-byte loads.  The (cos, sin) of a rotary pair (fp64 angle = fp64
// coordinate x fp64 inverse frequency, fp64 sincos, rounded to fp32) is shared
// by all heads and by Q and K, so each lane computes the few pairs it meets
// once per row, not per element.  Persistent grid, grid-stride over rows.
#pragma once

#include "common.cuh"

namespace h3 {

struct RopeTable {
  double inv_freq[64];   // per rotary pair
  int axis[64];          // 0 = t, 1 = h, 2 = w
};

constexpr int ROPE_THREADS = 256;
constexpr int ROPE_CTAS_PER_SM = 2;   // register-limited residency of rope_kernel

// (cos, sin) of pair p for a row with coordinates crd[0..2]: fp64 angle =
// fp64(coordinate) x fp64 inverse frequency, fp64 sincos, each rounded to fp32.
// Shared by the rope kernel and the attention kernel's fused Q rotation, so
// both produce identical rotated values.
__device__ __forceinline__ float2 rope_cos_sin(const RopeTable& tab, const float* crd, int p) {
  const double a = static_cast<double>(crd[tab.axis[p]]) * tab.inv_freq[p];
  double sn, cn;
  sincos(a, &sn, &cn);
  return make_float2(static_cast<float>(cn), static_cast<float>(sn));
}

// (x0, x1) -> (x0 c - x1 s, x0 s + x1 c) with every rounding explicit (no
// compiler-chosen contraction), so the result does not depend on the caller.
__device__ __forceinline__ void rot2(float x0, float x1, float2 cs, float& y0, float& y1) {
  y0 = __fmaf_rn(x0, cs.x, -__fmul_rn(x1, cs.y));
  y1 = __fmaf_rn(x0, cs.y, __fmul_rn(x1, cs.x));
}

// Rotate 4 adjacent pairs held in one 16-byte chunk (8 bf16).
__device__ __forceinline__ uint4 rotate_adjacent(uint4 v, const float2* cs) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&w[m]);
    float2 f = __bfloat1622float2(b);
    float y0, y1;
    rot2(f.x, f.y, cs[m], y0, y1);
    w[m] = pack_bf16x2(y0, y1);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Rotate 8 half-split pairs: chunk a holds x0 of pairs p..p+7, chunk b x1.
__device__ __forceinline__ void rotate_half(uint4& a, uint4& b, const float2* cs) {
  uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wa[m]));
    float2 fb = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wb[m]));
    float a0, b0, a1, b1;
    rot2(fa.x, fb.x, cs[2 * m], a0, b0);
    rot2(fa.y, fb.y, cs[2 * m + 1], a1, b1);
    wa[m] = pack_bf16x2(a0, a1);
    wb[m] = pack_bf16x2(b0, b1);
  }
  a = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  b = make_uint4(wb[0], wb[1], wb[2], wb[3]);
}

// The (cos, sin) of every rotary pair of every row, exactly as the rotation
// uses them: one thread per (row, pair), consecutive threads writing
// consecutive 8-byte entries of the [n_rows][64] table.
__global__ void __launch_bounds__(256) rope_cos_sin_kernel(const float* __restrict__ coords, long long n_rows,
                                                           float2* __restrict__ cs, const RopeTable tab) {
  const long long n = n_rows * 64;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    cs[i] = rope_cos_sin(tab, coords + 3 * (i >> 6), static_cast<int>(i & 63));
}

// One warp per packed row.  A row of one tensor is n_heads x 16 chunks of 16
// bytes; lane l handles the chunks (or, half-split, the chunk pairs) l, l + 32,
// ...  Because 32 is a multiple of the chunks per head, a lane always meets the
// same rotary pairs (4 adjacent pairs, or 8 half-split pairs) in every head, so
// it computes their (cos, sin) itself, once per row, while its first loads are
// in flight: no shared memory and no block barrier.  q / qo may both be null:
// then only K is rotated.  LAYOUT 0: pair p = dims (2p, 2p+1), one item = one
// chunk; LAYOUT 1: pair p = dims (p, p+64), one item = chunks c and c+8.
template <int LAYOUT>
__global__ void __launch_bounds__(ROPE_THREADS, ROPE_CTAS_PER_SM) rope_kernel(
    const uint4* q, const uint4* k, uint4* qo, uint4* ko, const float* __restrict__ coords,
    long long n_rows, int n_heads, long long stride16, const RopeTable tab) {
  constexpr int IPH = LAYOUT == 0 ? 16 : 8;        // work items per head
  constexpr int PPI = LAYOUT == 0 ? 4 : 8;         // rotary pairs per item
  constexpr int B = LAYOUT == 0 ? 7 : 4;           // items per lane in flight
  const int lane = threadIdx.x & 31;
  const int sub = lane % IPH;                      // item index within the head
  const long long gw = (static_cast<long long>(blockIdx.x) * ROPE_THREADS + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * ROPE_THREADS) >> 5;
  const int items = n_heads * IPH;
  const bool has_q = q != nullptr;
  for (long long r = gw; r < n_rows; r += nw) {
    const long long row_off = r * stride16;
    float2 cs[PPI];
    bool first = true;
    for (int i0 = lane; i0 < items; i0 += 32 * B) {
      uint4 qa[B], ka[B], qb[B], kb[B];
      long long off[B];
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int item = i0 + 32 * u;
        off[u] = -1;
        if (item < items) {
          off[u] = row_off + (item / IPH) * 16 + sub;
          if (has_q) qa[u] = __ldcs(q + off[u]);
          ka[u] = __ldcs(k + off[u]);
          if (LAYOUT == 1) {
            if (has_q) qb[u] = __ldcs(q + off[u] + 8);
            kb[u] = __ldcs(k + off[u] + 8);
          }
        }
      }
      if (first) {
        const float* crd = coords + 3 * r;
#pragma unroll
        for (int m = 0; m < PPI; ++m) cs[m] = rope_cos_sin(tab, crd, PPI * sub + m);
        first = false;
      }
#pragma unroll
      for (int u = 0; u < B; ++u) {
        if (off[u] < 0) continue;
        if (LAYOUT == 0) {
          if (has_q) __stcs(qo + off[u], rotate_adjacent(qa[u], cs));
          __stcs(ko + off[u], rotate_adjacent(ka[u], cs));
        } else {
          if (has_q) {
            rotate_half(qa[u], qb[u], cs);
            __stcs(qo + off[u], qa[u]);
            __stcs(qo + off[u] + 8, qb[u]);
          }
          rotate_half(ka[u], kb[u], cs);
          __stcs(ko + off[u], ka[u]);
          __stcs(ko + off[u] + 8, kb[u]);
        }
      }
    }
  }
}

}  // namespace h3
