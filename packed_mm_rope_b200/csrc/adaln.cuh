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
// Rows are staged in shared memory by bulk asynchronous copies (16 rows in
// flight per SM) and each warp owns a row at a time, so the statistics need
// only warp shuffles.
#pragma once

#include "common.cuh"

namespace h3 {

constexpr int ADALN_THREADS = 256;    // 8 warps, one row per warp at a time
constexpr int ADALN_WARPS = ADALN_THREADS / 32;
constexpr int ADALN_MAX_HIDDEN = 8192;

// Ring slots per warp: two when two rows per warp fit next to the table entry
// in shared memory, else one.
__host__ __device__ constexpr int adaln_slots(int hidden) { return hidden <= 5760 ? 2 : 1; }

// Dynamic shared memory: one cached table entry (shift then scale, fp32,
// 2 x hidden), then per warp adaln_slots(hidden) rows of x (bf16), then one
// mbarrier per warp slot.
__host__ __device__ constexpr size_t adaln_smem_bytes(int hidden) {
  return static_cast<size_t>(hidden) * 8 + static_cast<size_t>(ADALN_WARPS) * adaln_slots(hidden) * hidden * 2 +
         ADALN_WARPS * 2 * 8;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// CTA b owns the contiguous rows [b * per_cta, min(n, (b + 1) * per_cta));
// warp w of it takes every ADALN_WARPS-th of them.  Each warp streams its rows
// through its own ring (bulk copies issued by its lane 0), reduces mean and
// variance with shuffles only (no block barriers), and writes the modulated
// row with 16-byte stores.  The table entry of the CTA's first row is cached in
// shared memory; a row with another entry reads its entry from L2 directly.
__global__ void __launch_bounds__(ADALN_THREADS) adaln_kernel(
    const uint4* x, uint4* y, const int32_t* __restrict__ ts_idx, const int32_t* __restrict__ tags,
    const float4* __restrict__ table, int n_entries, long long n_rows, int chunks, long long x_stride16,
    long long y_stride16, float eps, unsigned long long wait_limit_ns, long long per_cta) {
  extern __shared__ __align__(16) uint8_t adaln_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hidden = chunks * 8;
  const int slots = adaln_slots(hidden);
  float4* entry_s = reinterpret_cast<float4*>(adaln_smem);
  uint4* ring = reinterpret_cast<uint4*>(adaln_smem + static_cast<size_t>(hidden) * 8) +
                static_cast<size_t>(warp) * slots * chunks;
  const uint32_t bar = smem_u32(adaln_smem + static_cast<size_t>(hidden) * 8 +
                                static_cast<size_t>(ADALN_WARPS) * slots * chunks * 16) + 16u * warp;
  const uint32_t row_bytes = static_cast<uint32_t>(chunks) * 16u;
  const float inv_c = 1.f / static_cast<float>(hidden);
  const long long r_begin = blockIdx.x * per_cta;
  const long long r_end = min(n_rows, r_begin + per_cta);
  if (r_begin >= r_end) return;

  // cached entry: that of the CTA's first row (a valid index, else none)
  const long long e0 = static_cast<long long>(ts_idx[r_begin]) * 3 + tags[r_begin];
  const bool e0_ok = e0 >= 0 && e0 < n_entries;
  // cached as (shift, 1 + scale)
  if (e0_ok)
    for (int i = threadIdx.x; i < 4 * chunks; i += ADALN_THREADS) {
      float4 t = table[e0 * 4LL * chunks + i];
      if (i >= 2 * chunks) t = make_float4(1.f + t.x, 1.f + t.y, 1.f + t.z, 1.f + t.w);
      entry_s[i] = t;
    }
  if (lane == 0)
    for (int i = 0; i < slots; ++i) mbar_init(bar + 8u * i, 1);
  mbar_fence_init();
  __syncthreads();

  // this warp's rows: r_begin + warp + k * ADALN_WARPS
  const long long first = r_begin + warp;
  const long long my_rows = first < r_end ? (r_end - first + ADALN_WARPS - 1) / ADALN_WARPS : 0;
  auto issue = [&](long long k) {
    const int slot = static_cast<int>(k % slots);
    mbar_arrive_expect_tx(bar + 8u * slot, row_bytes);
    bulk_load(smem_u32(ring + static_cast<size_t>(slot) * chunks), x + (first + k * ADALN_WARPS) * x_stride16,
              row_bytes, bar + 8u * slot);
  };
  if (lane == 0)
    for (long long k = 0; k < slots && k < my_rows; ++k) issue(k);
  uint32_t no_abort = 0u;
  long long k = 0;
  for (; k < my_rows; ++k) {
    const long long r = first + k * ADALN_WARPS;
    const int slot = static_cast<int>(k % slots);
    const bool landed = mbar_wait_bounded(bar + 8u * slot, static_cast<uint32_t>((k / slots) & 1), &no_abort,
                                          wait_limit_ns);
    if (!__all_sync(0xffffffffu, landed)) break;
    const uint4* row = ring + static_cast<size_t>(slot) * chunks;
    // One pass for both statistics, shifted by the row's first element to
    // avoid cancellation: mean = K + S1/n, var = S2/n - (S1/n)^2 with
    // S1 = sum(x - K), S2 = sum((x - K)^2).  Two elements per fp32x2 op.
    const float kf = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(row));
    const float2 k2 = make_float2(-kf, -kf);
    float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
    for (int c = lane; c < chunks; c += 32) {
      const uint4 u = row[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 d = __fadd2_rn(__bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[m])), k2);
        s1 = __fadd2_rn(s1, d);
        s2 = __ffma2_rn(d, d, s2);
      }
    }
    const float m1 = warp_sum(s1.x + s1.y) * inv_c;
    const float var = fmaxf(warp_sum(s2.x + s2.y) * inv_c - m1 * m1, 0.f);
    const float mean = kf + m1;
    const float rstd = rsqrtf(var + eps);
    const long long e = static_cast<long long>(ts_idx[r]) * 3 + tags[r];
    const bool bad = e < 0 || e >= n_entries;
    if (bad && lane == 0) atomicOr(&g_error_word, DEVERR_INPUT);
    const bool cached = e0_ok && e == e0;
    const float4* ent = cached ? entry_s : table + (bad ? 0 : e) * 4LL * chunks;
    const float one = cached ? 0.f : 1.f;           // the cache already holds 1 + scale
    // y = x * a + b with a = rstd * (1 + scale), b = shift - mean * a
    const float2 rs2 = make_float2(rstd, rstd), nm2 = make_float2(-mean, -mean), one2 = make_float2(one, one);
    for (int c = lane; c < chunks; c += 32) {
      const uint4 u = row[c];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      const float4 s0 = ent[2 * c], s1v = ent[2 * c + 1];
      const float4 g0 = ent[2 * chunks + 2 * c], g1 = ent[2 * chunks + 2 * c + 1];
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
      y[r * y_stride16 + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncwarp();                      // every lane has finished reading the slot
    if (lane == 0 && k + slots < my_rows) issue(k + slots);
  }
  // Drain: bulk copies this warp started land before the CTA exits (only
  // after an early exit are any still in flight).
  if (lane == 0) {
    volatile uint32_t never = 0u;
    const long long issued = my_rows < k + slots ? my_rows : k + slots;
    for (long long i = k; i < issued; ++i)
      mbar_wait_bounded(bar + 8u * static_cast<uint32_t>(i % slots), static_cast<uint32_t>((i / slots) & 1),
                        &never, 2000000000ull);
  }
}

}  // namespace h3
