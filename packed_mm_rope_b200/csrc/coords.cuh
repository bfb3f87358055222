// coords.cuh -- packed segment table -> per-row (t, h, w) fp32 coordinates.
//
// "Inside MiniMax H3" section 4: three-axis positions on one physical
// timeline; stereo channels share t and differ on another axis; packed row
// order carries no position.  "MiniMax H3 -- one transformer that denoises
// video and audio together": every token of a latent frame has that frame's
// t and differs only in (h, w); text t is the token index; one clock unit is
// one audio latent (1/40 s).
//
// One thread per packed row: look up the logical element (through the
// optional permutation), find its segment by binary search over the prefix
// row counts, decode the element index, and form t as ONE IEEE division of
// two exactly representable integers, so t is the correctly rounded quotient.
#pragma once

#include "common.cuh"

namespace h3 {

struct CoordTable {
  h3_segment seg[H3_MAX_SEGMENTS];
  long long first[H3_MAX_SEGMENTS + 1];   // first logical row of each segment
  int nseg;
};

__device__ __forceinline__ float exact_ratio(long long num, int den) {
  // |num| < 2^24 and 0 < den < 2^24 are checked on the host, so both
  // conversions are exact and __fdiv_rn rounds the true quotient once.
  return __fdiv_rn(static_cast<float>(num), static_cast<float>(den));
}

// Normalised spatial canvas ("MiniMax H3 -- one transformer ...", passage on
// resolution: the grid is normalised by sqrt(H W) and centred on [0, 32)):
//   16 + (idx + 1/2 - n/2) * 32 / sqrt(H W)
// evaluated in fp64 one IEEE operation at a time (explicit _rn intrinsics, so
// nothing is contracted into an FMA), then rounded to fp32.
__device__ __forceinline__ float canvas(long long idx, int n, int gh, int gw) {
  const double a = __dadd_rn(static_cast<double>(idx), 0.5);
  const double b = __dsub_rn(a, __dmul_rn(0.5, static_cast<double>(n)));
  const double s = __ddiv_rn(32.0, __dsqrt_rn(__dmul_rn(static_cast<double>(gh), static_cast<double>(gw))));
  return __double2float_rn(__dadd_rn(16.0, __dmul_rn(b, s)));
}

__global__ void __launch_bounds__(256) coords_kernel(const CoordTable tab, const int32_t* perm,
                                                     long long n_rows, float* out, int err_slot) {
  const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; r < n_rows;
       r += step) {
    long long e = r;
    if (perm != nullptr) {
      e = perm[r];
      if (e < 0 || e >= n_rows) {
        raise_error(err_slot, DEVERR_INPUT);
        const float nan = __int_as_float(0x7fc00000);
        out[3 * r + 0] = nan;
        out[3 * r + 1] = nan;
        out[3 * r + 2] = nan;
        continue;
      }
    }
    // largest s with first[s] <= e; that segment is non-empty and holds e
    int lo = 0, hi = tab.nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab.first[mid] <= e) lo = mid; else hi = mid - 1;
    }
    const h3_segment& s = tab.seg[lo];
    const long long local = e - tab.first[lo];
    float t, h, w;
    if (s.kind == H3_SEG_TEXT) {
      t = exact_ratio(s.t_off_num + local * s.t_step_num, s.t_den);
      const bool t_only = (s.flags & H3_FLAG_TEXT_T_ONLY) != 0;
      h = t_only ? 0.f : t;
      w = t_only ? 0.f : t;
    } else if (s.kind == H3_SEG_VIDEO) {
      const long long per_frame = static_cast<long long>(s.grid_h) * s.grid_w;
      const long long k = local / per_frame;
      const long long cell = local - k * per_frame;
      const long long y = cell / s.grid_w;
      const long long x = cell - y * s.grid_w;
      t = exact_ratio(s.t_off_num + k * s.t_step_num, s.t_den);
      if (s.flags & H3_FLAG_VIDEO_CANVAS) {
        h = canvas(y, s.grid_h, s.grid_h, s.grid_w);
        w = canvas(x, s.grid_w, s.grid_h, s.grid_w);
      } else {
        h = static_cast<float>(y);
        w = static_cast<float>(x);
      }
    } else {  // H3_SEG_AUDIO
      const long long j = local / s.channels;
      const float c = static_cast<float>(local - j * s.channels);
      t = exact_ratio(s.t_off_num + j * s.t_step_num, s.t_den);
      const bool on_h = (s.flags & H3_FLAG_AUDIO_CHANNEL_H) != 0;
      h = on_h ? c : 0.f;
      w = on_h ? 0.f : c;
    }
    out[3 * r + 0] = t;
    out[3 * r + 1] = h;
    out[3 * r + 2] = w;
  }
}

}  // namespace h3
