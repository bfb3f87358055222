// rope.cuh -- fused three-axis MM-RoPE rotation of bf16 Q and K.
//
// "Inside MiniMax H3" section 4 and the model card's H3-Omni-Transformer
// section: Q and K are rotated by a (t, h, w) rotary embedding; the explainer
// page traces position_ids[:, 0] (t) into rope() and the rotation of Q and K,
// with inverse frequencies computed from rope_theta / rope_freq_dim.
//
// HBM-bound streaming kernel.  A CTA owns ROWS packed rows at a time: it
// first builds the 64 (cos, sin) pairs of each row in shared memory (fp64
// angle = fp64 coordinate x fp64 inverse frequency, fp64 sincos, rounded to
// fp32), then streams both tensors with 16-byte loads.  The angles of a row
// are shared by all heads and by Q and K, so the trigonometry is paid once
// per row, not per element.  Persistent grid, grid-stride over row blocks.
#pragma once

#include "common.cuh"

namespace h3 {

struct RopeTable {
  double inv_freq[64];   // per rotary pair
  int axis[64];          // 0 = t, 1 = h, 2 = w
};

constexpr int ROPE_THREADS = 256;
constexpr int ROPE_ROWS = 8;      // rows per block iteration
constexpr int ROPE_UNROLL = 4;    // independent 16-byte chunks in flight per thread

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

// q / qo may both be null: then only K is rotated.
// LAYOUT 0: pair p = dims (2p, 2p+1); one work item = one 16-byte chunk.
// LAYOUT 1: pair p = dims (p, p+64);  one work item = chunks c and c+8 of a head.
template <int LAYOUT>
__global__ void __launch_bounds__(ROPE_THREADS) rope_kernel(
    const uint4* q, const uint4* k, uint4* qo, uint4* ko, const float* __restrict__ coords,
    long long n_rows, int n_heads, long long stride16, const RopeTable tab) {
  __shared__ float2 cs[ROPE_ROWS][64];
  constexpr int ITEMS_PER_HEAD = LAYOUT == 0 ? 16 : 8;
  const int items_per_row = n_heads * ITEMS_PER_HEAD;
  const long long nblk = (n_rows + ROPE_ROWS - 1) / ROPE_ROWS;

  for (long long blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
    const long long r0 = blk * ROPE_ROWS;
    const int nr = static_cast<int>(min(static_cast<long long>(ROPE_ROWS), n_rows - r0));
    __syncthreads();   // previous block's readers are done with cs
    for (int i = threadIdx.x; i < nr * 64; i += ROPE_THREADS) {
      const int r = i >> 6, p = i & 63;
      cs[r][p] = rope_cos_sin(tab, coords + 3 * (r0 + r), p);
    }
    __syncthreads();

    const int total = nr * items_per_row;
    for (int base = threadIdx.x; base < total; base += ROPE_THREADS * ROPE_UNROLL) {
      uint4 qa[ROPE_UNROLL], ka[ROPE_UNROLL], qb[ROPE_UNROLL], kb[ROPE_UNROLL];
      long long off[ROPE_UNROLL];
      int pair0[ROPE_UNROLL], row[ROPE_UNROLL];
#pragma unroll
      for (int u = 0; u < ROPE_UNROLL; ++u) {
        const int item = base + u * ROPE_THREADS;
        off[u] = -1;
        if (item < total) {
          const int r = item / items_per_row;
          const int c = item - r * items_per_row;
          const int head = c / ITEMS_PER_HEAD;
          const int sub = c - head * ITEMS_PER_HEAD;
          row[u] = r;
          off[u] = (r0 + r) * stride16 + head * 16 + sub;
          pair0[u] = LAYOUT == 0 ? 4 * sub : 8 * sub;
          if (q != nullptr) qa[u] = __ldcs(q + off[u]);
          ka[u] = __ldcs(k + off[u]);
          if (LAYOUT == 1) {
            if (q != nullptr) qb[u] = __ldcs(q + off[u] + 8);
            kb[u] = __ldcs(k + off[u] + 8);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < ROPE_UNROLL; ++u) {
        if (off[u] < 0) continue;
        const float2* c = &cs[row[u]][pair0[u]];
        if (LAYOUT == 0) {
          if (q != nullptr) __stcs(qo + off[u], rotate_adjacent(qa[u], c));
          __stcs(ko + off[u], rotate_adjacent(ka[u], c));
        } else {
          if (q != nullptr) {
            rotate_half(qa[u], qb[u], c);
            __stcs(qo + off[u], qa[u]);
            __stcs(qo + off[u] + 8, qb[u]);
          }
          rotate_half(ka[u], kb[u], c);
          __stcs(ko + off[u], ka[u]);
          __stcs(ko + off[u] + 8, kb[u]);
        }
      }
    }
  }
}

}  // namespace h3
