// attention.cuh -- full softmax attention over one packed sequence (sm_100a).
//
// "Inside MiniMax H3" sections 2 and 6: every modality's rows share one
// attention sequence and the open inference path runs FULL attention, whose
// cost dominates long videos; "MiniMax H3 -- one transformer ..." notes that
// attention is bidirectional.  So: O = softmax(Q K^T * scale) V per (batch,
// head), no mask, every row attends to every row.
//
// Design (one CTA per 256 query rows of one head, one CTA per SM):
//   warps 0-3   softmax warpgroup for query tile 0 (rows   0..127)
//   warps 4-7   softmax warpgroup for query tile 1 (rows 128..255)
//   warp  8     TMA producer: Q tiles once, then K_j, V_j into a ring
//   warp  9     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128)  S0 = Q0 K_j^T    (P0 = bf16 softmax numerators aliased on
//   [128,256)  S1 = Q1 K_j^T     its first 64 columns, two per column)
//   [256,384)  O0 accumulator   [384,512) O1 accumulator
// Per KV tile j the issuer runs  PV0(j), S0(j+1), PV1(j), S1(j+1): while one
// warpgroup exponentiates its S tile the tensor core works on the other.  Each
// P tile is released in two 64-key halves with their own barriers, so the
// first half of P.V runs while the second half is still being exponentiated.
//
// Softmax (one thread = one query row, the row lives in one TMEM lane):
// logits are handled in log2 units (x = s * scale * log2 e).  Numerators are
// 2^(x - m) against a running reference m that is only raised when a 64-key
// half would overflow the headroom: the half's numerators are computed first
// (speculatively, against the current m) and kept unless their sum exceeds
// 2^64.  Then the half's true maximum is taken, O (in TMEM) and the row sum
// are multiplied by 2^(m_old - m_new), and the half is recomputed.  Any m
// gives the same quotient O / l; the limit only keeps numerators, sums and O
// far from fp32/bf16 overflow.  In practice m is set by the first half-tile
// and never moves again, so the hot loop has no max reduction at all: one
// packed fp32x2 FMA, two MUFU ex2, one packed add and one bf16x2 conversion per
// pair of logits.  The S tile of step j+1 is only issued after PV(j), so when
// a warpgroup sees S(j) complete, O already holds PV(j-1) and a rescale for
// the first half can be applied in place; a rescale for the second half first
// waits for the first half of PV(j) to land (pva_done).
//
// Shared memory (1024-byte aligned): Q0, Q1 (32 KB each) and a ring of
// KV_STAGES 32 KB slots; every 128 x 128 bf16 tile is two 128-row x 64-column
// halves in the TMA 128-byte-swizzle layout, which is the canonical K-major
// layout for Q and K and the MN-major layout for V as a B operand.
//
// Every mbarrier wait is bounded (global-time limit); a thread that gives up
// raises an abort flag that all other waits observe, the producer and the
// issuer drain what they already started, and TMEM is freed before exit.
#pragma once

#include "common.cuh"
#include "rope.cuh"

namespace h3 {
namespace attn {

constexpr int BM = 128;          // query rows per tile (MMA M)
constexpr int BN = 128;          // key rows per tile  (S MMA N, PV MMA K)
constexpr int HD = 128;          // head dim
constexpr int KV_STAGES = 4;     // K/V ring slots of 32 KB
constexpr int THREADS = 320;
constexpr uint32_t TILE_BYTES = BM * HD * 2;     // 32768
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;  // 16384
constexpr float SUM_LIMIT = 18446744073709551616.0f;   // 2^64

constexpr uint32_t SMEM_Q = 0;
constexpr uint32_t SMEM_KV = 2 * TILE_BYTES;
constexpr uint32_t SMEM_BAR = SMEM_KV + KV_STAGES * TILE_BYTES;
// barriers: q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2][2] (halves),
//           pva_done[2] (first half of PV landed), o_full[2], mma_done,
//           q_ready[2] (Q tile rotated in place, fused RoPE only)
constexpr int NUM_BARS = 2 + 2 * KV_STAGES + 2 + 4 + 2 + 2 + 1 + 2;
constexpr uint32_t SMEM_MISC = SMEM_BAR + NUM_BARS * 8;   // tmem base, abort flag
constexpr uint32_t SMEM_BYTES = SMEM_MISC + 16 + 1024;    // + alignment slack

constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);   // Q, K both K-major
constexpr uint32_t IDESC_O = idesc_bf16_f32(BM, HD, false, true);    // P from TMEM, V MN-major

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S0 = 0, TMEM_O0 = 256;

// Waits of the single MMA-issuing thread spin with test_wait (never suspend):
// it is on the critical path of both query tiles.
__device__ __forceinline__ bool mma_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                         uint64_t limit, int err_slot) {
  return mbar_spin_bounded(bar, parity, abort, limit, err_slot);
}

// All lanes wait; the warp proceeds only if every lane saw the phase complete,
// so the .sync.aligned tcgen05 instructions that follow run converged.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                          uint64_t limit, int err_slot) {
  const bool r = mbar_wait_bounded(bar, parity, abort, limit, err_slot);
  return __all_sync(0xffffffffu, r);
}

struct Params {
  int n_rows;
  int n_heads;
  int n_kv_tiles;
  float scale_log2;               // softmax scale * log2(e)
  __nv_bfloat16* o;
  long long o_row_stride;         // elements
  long long o_batch_stride;       // elements
  float* lse;                     // [B][H][N] or null
  unsigned long long wait_limit_ns;
  unsigned long long drain_limit_ns;
  int err_slot;                   // error word of the launching stream
  // fused RoPE on Q (rope_cs == null: Q arrives rotated)
  const float2* rope_cs;          // [B][N][64] (cos, sin) per rotary pair
  int rope_layout;                // 0 adjacent pairs, 1 half-split
};

// 2^(x*sl2 - m) for 64 logits: bf16 pairs and their sum.  Two logits per
// packed fp32x2 FMA and add (Blackwell f32x2 arithmetic) keep the instruction
// count per element at 2.5: the softmax warps are issue-bound, not MUFU-bound.
__device__ __forceinline__ void exp_half(const float (&x)[64], float sl2, float m, uint32_t (&pk)[32],
                                         float& ls) {
  const float2 c2 = make_float2(sl2, sl2), mm = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const float2 y = __ffma2_rn(make_float2(x[2 * c], x[2 * c + 1]), c2, mm);
    const float p0 = ex2_approx(y.x), p1 = ex2_approx(y.y);
    acc[c & 3] = __fadd2_rn(acc[c & 3], make_float2(p0, p1));
    pk[c] = pack_bf16x2(p0, p1);
  }
  const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  ls = t.x + t.y;
}

// Raw maximum of 64 logits (only on the rare rescale path).
__device__ __forceinline__ float max64(const float (&x)[64]) {
  float ma[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ma[i] = x[i];
#pragma unroll
  for (int c = 8; c < 64; ++c) ma[c & 7] = fmaxf(ma[c & 7], x[c]);
  return fmaxf(fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3])), fmaxf(fmaxf(ma[4], ma[5]), fmaxf(ma[6], ma[7])));
}

__global__ void __launch_bounds__(THREADS, 1)
attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - raw);

  const uint32_t bar0 = base + SMEM_BAR;
  auto bar_q_full = [&](int i) { return bar0 + 8u * i; };
  auto bar_kv_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto bar_kv_empty = [&](int s) { return bar0 + 8u * (2 + KV_STAGES + s); };
  auto bar_s_full = [&](int i) { return bar0 + 8u * (2 + 2 * KV_STAGES + i); };
  auto bar_p_full = [&](int i, int half) { return bar0 + 8u * (4 + 2 * KV_STAGES + 2 * i + half); };
  auto bar_pva_done = [&](int i) { return bar0 + 8u * (8 + 2 * KV_STAGES + i); };
  auto bar_o_full = [&](int i) { return bar0 + 8u * (10 + 2 * KV_STAGES + i); };
  const uint32_t bar_mma_done = bar0 + 8u * (12 + 2 * KV_STAGES);
  auto bar_q_ready = [&](int i) { return bar0 + 8u * (13 + 2 * KV_STAGES + i); };
  const bool fused_rope = p.rope_cs != nullptr;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gbase + SMEM_MISC);
  volatile uint32_t* const abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + SMEM_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int batch = blockIdx.z;
  const int q_row0 = blockIdx.x * (2 * BM);
  const int nkv = p.n_kv_tiles;
  const uint64_t limit = p.wait_limit_ns;
  const int eslot = p.err_slot;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_q_full(i), 1);
      mbar_init(bar_s_full(i), 1);
      mbar_init(bar_p_full(i, 0), 128);
      mbar_init(bar_p_full(i, 1), 128);
      mbar_init(bar_pva_done(i), 1);
      mbar_init(bar_o_full(i), 1);
    }
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_mma_done, 1);
    mbar_init(bar_q_ready(0), 128);
    mbar_init(bar_q_ready(1), 128);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA ----
    if (lane == 0) {
      const int col0 = head * HD;
      for (int i = 0; i < 2; ++i) {
        const uint32_t dst = base + SMEM_Q + i * TILE_BYTES;
        mbar_arrive_expect_tx(bar_q_full(i), TILE_BYTES);
        tma_load_3d(dst, &tm_q, bar_q_full(i), col0, q_row0 + i * BM, batch);
        tma_load_3d(dst + HALF_BYTES, &tm_q, bar_q_full(i), col0 + 64, q_row0 + i * BM, batch);
      }
      int issued = 0;
      for (int idx = 0; idx < 2 * nkv; ++idx) {
        const int s = idx % KV_STAGES;
        const int use = idx / KV_STAGES;
        if (use > 0 && !mbar_wait_bounded(bar_kv_empty(s), (use - 1) & 1, abort_flag, limit, eslot)) break;
        const CUtensorMap* tm = (idx & 1) ? &tm_v : &tm_k;
        const int row = (idx >> 1) * BN;
        const uint32_t dst = base + SMEM_KV + s * TILE_BYTES;
        mbar_arrive_expect_tx(bar_kv_full(s), TILE_BYTES);
        tma_load_3d(dst, tm, bar_kv_full(s), col0, row, batch);
        tma_load_3d(dst + HALF_BYTES, tm, bar_kv_full(s), col0 + 64, row, batch);
        issued = idx + 1;
      }
      // Drain: every load this thread started must land before the CTA exits.
      // The drain ignores the abort flag (a never-raised local flag).
      volatile uint32_t never = 0u;
      for (int i = 0; i < 2; ++i) mbar_wait_bounded(bar_q_full(i), 0, &never, p.drain_limit_ns, eslot);
      for (int idx = (issued > KV_STAGES ? issued - KV_STAGES : 0); idx < issued; ++idx)
        mbar_wait_bounded(bar_kv_full(idx % KV_STAGES), (idx / KV_STAGES) & 1, &never,
                          p.drain_limit_ns, eslot);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA ----
    if (lane == 0) {
      auto q_addr = [&](int i) { return base + SMEM_Q + i * TILE_BYTES; };
      auto kv_addr = [&](int s) { return base + SMEM_KV + s * TILE_BYTES; };
      // S_i = Q_i K^T : 8 MMAs of K=16 over the two 64-column swizzled halves
      auto issue_s = [&](int i, int ks) {
        const uint32_t d = tmem + TMEM_S0 + i * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          mma_ss(d, smem_desc_sw128(q_addr(i) + off, 16, 1024),
                 smem_desc_sw128(kv_addr(ks) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // O_i += P_i V over keys [64*half, 64*half + 64): A = P_i from TMEM (8
      // columns per K=16 step), B = V rows from shared memory, MN-major
      auto issue_pv = [&](int i, int vs, int half, bool acc) {
        const uint32_t d = tmem + TMEM_O0 + i * 128;
        const uint32_t a = tmem + TMEM_S0 + i * 128;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * half + k4;
          mma_ts(d, a + kk * 8, smem_desc_sw128(kv_addr(vs) + kk * 2048, HALF_BYTES, 1024),
                 IDESC_O, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // P_i(j) in two halves; the first half's completion is announced on pva_done.
      // x (non-zero): a barrier the caller needs next, polled together with the
      // second half of P so that the two polls' latencies overlap
      auto issue_pv_tile = [&](int i, int vs, int j, uint32_t x, uint32_t x_par) -> bool {
        if (!mma_wait(bar_p_full(i, 0), j & 1, abort_flag, limit, eslot)) return false;
        tc_fence_after();
        issue_pv(i, vs, 0, j > 0);
        tc_commit(bar_pva_done(i));
        if (x != 0u ? !mbar_spin2_bounded(bar_p_full(i, 1), j & 1, x, x_par, abort_flag, limit, eslot)
                    : !mma_wait(bar_p_full(i, 1), j & 1, abort_flag, limit, eslot))
          return false;
        tc_fence_after();
        issue_pv(i, vs, 1, true);
        return true;
      };
      // with fused RoPE the softmax warpgroups rotate Q in place first
      auto bar_q = [&](int i) { return fused_rope ? bar_q_ready(i) : bar_q_full(i); };
      bool ok = mma_wait(bar_q(0), 0, abort_flag, limit, eslot) &&
                mma_wait(bar_kv_full(0), 0, abort_flag, limit, eslot);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        tc_commit(bar_s_full(0));
        ok = mma_wait(bar_q(1), 0, abort_flag, limit, eslot);
      }
      if (ok) {
        tc_fence_after();
        issue_s(1, 0);
        tc_commit(bar_s_full(1));
        tc_commit(bar_kv_empty(0));
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int vidx = 2 * j + 1, vs = vidx % KV_STAGES;
        const int kidx = 2 * j + 2, ks = kidx % KV_STAGES;
        const bool more = j + 1 < nkv;
        if (!mma_wait(bar_kv_full(vs), (vidx / KV_STAGES) & 1, abort_flag, limit, eslot)) break;
        // K(j + 1) is waited for together with the second half of P0(j): the chain
        // P0(j) -> P.V -> S0(j + 1) -> softmax pays one poll instead of two
        if (!issue_pv_tile(0, vs, j, more ? bar_kv_full(ks) : 0u, (kidx / KV_STAGES) & 1)) break;
        if (more) {
          tc_fence_after();
          issue_s(0, ks);
          tc_commit(bar_s_full(0));
        } else {
          tc_commit(bar_o_full(0));
        }
        if (!issue_pv_tile(1, vs, j, 0u, 0u)) break;
        tc_commit(bar_kv_empty(vs));
        if (more) {
          issue_s(1, ks);
          tc_commit(bar_s_full(1));
          tc_commit(bar_kv_empty(ks));
        } else {
          tc_commit(bar_o_full(1));
        }
      }
      // Drain: all MMAs issued above complete before TMEM is released.
      tc_commit(bar_mma_done);
      volatile uint32_t never = 0u;
      mma_wait(bar_mma_done, 0, &never, p.drain_limit_ns, eslot);
    }
  } else {
    // -------------------------------------------------------- softmax ----
    const int wg = warp >> 2;                      // query tile 0 or 1
    const int row_in_tile = threadIdx.x & 127;     // == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + TMEM_S0 + wg * 128;
    const uint32_t t_o = tmem + lane_base + TMEM_O0 + wg * 128;
    const float sl2 = p.scale_log2;
    const int tail = p.n_rows - (nkv - 1) * BN;    // valid keys in the last tile (1..128)
    float m_used = -INFINITY;                      // log2 units
    float l_sum = 0.f;
    bool ok = true;

    // registers of two TMEM chunks -> 64 logits; keys past the end -> -inf
    auto to_logits = [&](const uint32_t (&r)[2][32], int col0, bool last, float (&x)[64]) {
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(r[c >> 5][c & 31]);
      if (last && tail < BN) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (col0 + c >= tail) x[c] = -INFINITY;
      }
    };
    // O *= f for this warp's rows (warp-collective TMEM round trip)
    auto rescale_o = [&](float f) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + 32 * c, o);
        tmem_wait_ld(o);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
        tmem_st32(t_o + 32 * c, o);
      }
    };
    // Publish 64 keys of P (32 TMEM columns, aliasing the S columns already read).
    auto store_p = [&](int half, const uint32_t (&pk)[32]) {
      __syncwarp();
      tmem_st32(t_s + 32 * half, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full(wg, half));
    };

    // Fused RoPE: rotate this warpgroup's Q tile in shared memory, one thread
    // per row, with the (cos, sin) the rope kernel uses (read from the table)
    // and its rot2 arithmetic, then make the generic-proxy writes visible to
    // the tensor core (async proxy).
    if (fused_rope) {
      if (!warp_wait(bar_q_full(wg), 0, abort_flag, limit, eslot)) ok = false;
      const int row = q_row0 + wg * BM + row_in_tile;
      if (ok && row < p.n_rows) {
        const float4* cs4 = reinterpret_cast<const float4*>(p.rope_cs + (static_cast<long long>(batch) * p.n_rows + row) * 64);
        uint8_t* qrow = gbase + SMEM_Q + wg * TILE_BYTES + row_in_tile * 128;
        const int sw = row_in_tile & 7;           // 128-byte swizzle of this row
        auto chunk = [&](int c) {                 // logical 16-byte chunk c of 16
          return reinterpret_cast<uint4*>(qrow + (c >> 3) * HALF_BYTES + (((c & 7) ^ sw) << 4));
        };
        if (p.rope_layout == 0) {
#pragma unroll 4
          for (int c = 0; c < 16; ++c) {          // pairs 4c .. 4c+3
            const float4 a = __ldg(cs4 + 2 * c), b = __ldg(cs4 + 2 * c + 1);
            const float2 cs[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y),
                                  make_float2(b.z, b.w)};
            *chunk(c) = rotate_adjacent(*chunk(c), cs);
          }
        } else {
#pragma unroll 2
          for (int c = 0; c < 8; ++c) {           // pairs 8c .. 8c+7
            float2 cs[8];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const float4 a = __ldg(cs4 + 4 * c + m);
              cs[2 * m] = make_float2(a.x, a.y);
              cs[2 * m + 1] = make_float2(a.z, a.w);
            }
            uint4 a = *chunk(c), b = *chunk(c + 8);
            rotate_half(a, b, cs);
            *chunk(c) = a;
            *chunk(c + 8) = b;
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar_q_ready(wg));
    }

    for (int j = 0; j < nkv; ++j) {
      if (!warp_wait(bar_s_full(wg), j & 1, abort_flag, limit, eslot)) { ok = false; break; }
      tc_fence_after();
      const bool last = j == nkv - 1;
      float ls_a;
      {
        // ---- keys 0..63 ----
        uint32_t ra[2][32];
        tmem_ld32(t_s, ra[0]);
        tmem_ld32(t_s + 32, ra[1]);
        tmem_wait_ld(ra[0]);
        tmem_wait_ld(ra[1]);
        float xa[64];
        to_logits(ra, 0, last, xa);
        uint32_t pka[32];
        exp_half(xa, sl2, m_used, pka, ls_a);         // speculative against m_used
        const bool need = (j == 0) || !(ls_a <= SUM_LIMIT);
        if (__any_sync(0xffffffffu, need)) {
          float f = 1.f;
          if (need) {
            const float m_new = fmaxf(m_used, max64(xa) * sl2);
            f = (j == 0) ? 0.f : ex2_approx(m_used - m_new);
            m_used = m_new;
            l_sum *= f;
          }
          __syncwarp();
          if (j > 0) rescale_o(f);      // O holds PV(j-1); PV(j) has not started
          exp_half(xa, sl2, m_used, pka, ls_a);
        }
        l_sum += ls_a;
        store_p(0, pka);
      }
      {
        // ---- keys 64..127 ----
        uint32_t rb[2][32];
        __syncwarp();
        tmem_ld32(t_s + 64, rb[0]);
        tmem_ld32(t_s + 96, rb[1]);
        tmem_wait_ld(rb[0]);
        tmem_wait_ld(rb[1]);
        float xb[64];
        to_logits(rb, 64, last, xb);
        uint32_t pkb[32];
        float ls_b;
        exp_half(xb, sl2, m_used, pkb, ls_b);
        const bool need = !(ls_b <= SUM_LIMIT);
        if (__any_sync(0xffffffffu, need)) {
          // the first half of PV(j) may be in flight: let it land, then rescale
          // O (which now includes it) together with the running sum
          if (!warp_wait(bar_pva_done(wg), j & 1, abort_flag, limit, eslot)) { ok = false; break; }
          tc_fence_after();
          float f = 1.f;
          if (need) {
            const float m_new = fmaxf(m_used, max64(xb) * sl2);
            f = ex2_approx(m_used - m_new);
            m_used = m_new;
            l_sum *= f;
          }
          __syncwarp();
          rescale_o(f);
          exp_half(xb, sl2, m_used, pkb, ls_b);
        }
        l_sum += ls_b;
        store_p(1, pkb);
      }
    }

    // epilogue: O / l -> bf16 -> global; optional log-sum-exp
    if (ok && warp_wait(bar_o_full(wg), 0, abort_flag, limit, eslot)) {
      tc_fence_after();
      const int row = q_row0 + wg * BM + row_in_tile;
      const float inv_l = 1.f / l_sum;
      __nv_bfloat16* orow = p.o + batch * p.o_batch_stride + static_cast<long long>(row) * p.o_row_stride +
                            head * HD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld32(t_o + 32 * c, o);
        tmem_wait_ld(o);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (row < p.n_rows) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (p.lse != nullptr && row < p.n_rows) {
        p.lse[(static_cast<long long>(batch) * p.n_heads + head) * p.n_rows + row] =
            (m_used + __log2f(l_sum)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn
}  // namespace h3
