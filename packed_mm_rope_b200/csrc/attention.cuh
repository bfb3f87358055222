// attention.cuh -- full softmax attention over one packed sequence (sm_100a).
//
// "Inside MiniMax H3" sections 2 and 6: every modality's rows share one
// attention sequence and the open inference path runs FULL attention, whose
// cost dominates long videos; "MiniMax H3 -- one transformer ..." notes that
// attention is bidirectional.  So: O = softmax(Q K^T * scale) V per (batch,
// head), no mask, every row attends to every row.
//
// Design (one CTA per 256 query rows of one head, one CTA per SM):
//   warps 0-7   softmax for query tile 0 (rows   0..127)
//   warps 8-15  softmax for query tile 1 (rows 128..255)
//   warp  16    TMA producer: Q tiles once, then K_j, V_j into a ring
//   warp  17    TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128)  S0 = Q0 K_j^T    (P0 = bf16 softmax numerators aliased on
//   [128,256)  S1 = Q1 K_j^T     its first 64 columns, two per column)
//   [256,384)  O0 accumulator   [384,512) O1 accumulator
// Per KV tile j the issuer runs  PV0(j), S0(j+1), PV1(j), S1(j+1): while one
// query tile's warps exponentiate their S tile the tensor core works on the
// other.  Each P tile is released in two 64-key halves with their own
// barriers, so the first half of P.V runs while the second half is still being
// exponentiated.  The issuing thread polls V(j) together with the first half of
// P0(j) and K(j+1) together with its second half: one barrier poll whose result
// is branched on costs it ~160 cycles, and the second pair sits on the chain
// P0(j) -> P.V -> S0(j+1) -> softmax.
//
// Softmax: four threads per query row.  Warp w of a query tile reads the 16
// TMEM lanes 32 (w % 4) + 16 ((w / 4) % 2) + [0, 16) with the 16x256b shape,
// so thread (t0 = lane % 4, t1 = lane / 4) holds rows t1 and t1 + 8 of those
// lanes and, of every 8-column block, columns 2 t0 and 2 t0 + 1; the four
// threads of a row (a quad) together hold its 128 keys.  Four warps per
// sub-partition hide each other's TMEM and barrier latencies (one thread per
// row leaves two).  Logits are handled in log2 units (x = s * scale * log2 e).
// Numerators are 2^(x - m) against a running reference m per row that is only
// raised when a thread's share of a 64-key half would overflow the headroom:
// the half's numerators are computed first (speculatively, against the current
// m) and kept unless a share exceeds 2^62 (four shares stay below 2^64).  Then
// the quad takes the half's true maximum by shuffles, O (in TMEM) and the row
// sums are multiplied by 2^(m_old - m_new), and the half is recomputed.  Any m
// gives the same quotient O / l; the limit only keeps numerators, sums and O
// far from fp32/bf16 overflow.  In practice m is set by the first half-tile
// and never moves again, so the hot loop has no max reduction at all: one
// packed fp32x2 FMA, two MUFU ex2, one packed add and one bf16x2 conversion per
// pair of logits.  The S tile of step j+1 is only issued after PV(j), so when
// a warp sees S(j) complete, O already holds PV(j-1) and a rescale for the
// first half can be applied in place; a rescale for the second half first
// waits for the first half of PV(j) to land (pva_done).  Each thread keeps its
// share of the row sums; the quad adds them once, in the epilogue.
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
constexpr int SOFTMAX_WARPS = 16;                   // 8 per query tile, four threads per row
constexpr int W_PROD = SOFTMAX_WARPS;                // TMA producer
constexpr int W_MMA = SOFTMAX_WARPS + 1;             // TMEM allocator and MMA issuer
constexpr int THREADS = 32 * (SOFTMAX_WARPS + 2);    // 576
constexpr uint32_t TILE_BYTES = BM * HD * 2;     // 32768
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;  // 16384

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
      mbar_init(bar_p_full(i, 0), 8);    // one arrival per softmax warp of the tile
      mbar_init(bar_p_full(i, 1), 8);
      mbar_init(bar_pva_done(i), 1);
      mbar_init(bar_o_full(i), 1);
    }
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    mbar_init(bar_mma_done, 1);
    mbar_init(bar_q_ready(0), 8);
    mbar_init(bar_q_ready(1), 8);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == W_PROD && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == W_PROD) {
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
  } else if (warp == W_MMA) {
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
      // x / y (non-zero): a barrier the caller needs, polled together with the
      // second / first half of P so that the two polls' latencies overlap
      auto issue_pv_tile = [&](int i, int vs, int j, uint32_t x, uint32_t x_par, uint32_t y = 0u,
                               uint32_t y_par = 0u) -> bool {
        if (y != 0u ? !mbar_spin2_bounded(bar_p_full(i, 0), j & 1, y, y_par, abort_flag, limit, eslot)
                    : !mma_wait(bar_p_full(i, 0), j & 1, abort_flag, limit, eslot))
          return false;
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
        // V(j) is waited for together with the first half of P0(j), K(j + 1)
        // together with its second half
        if (!issue_pv_tile(0, vs, j, more ? bar_kv_full(ks) : 0u, (kidx / KV_STAGES) & 1, bar_kv_full(vs),
                           (vidx / KV_STAGES) & 1))
          break;
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
    // Eight warps per query tile, four threads per row: warp w reads the 16
    // TMEM lanes 32 (w % 4) + 16 ((w / 4) % 2) + [0, 16) with the 16x256b
    // shape, so thread (t0 = lane % 4, t1 = lane / 4) holds rows t1 and t1 + 8
    // of that group and, of every 8-column block, columns 2 t0 and 2 t0 + 1.
    // The four threads of a row agree on its reference through shuffles.
    const int wg = warp >> 3;                      // query tile 0 or 1
    const int t0 = lane & 3, t1 = lane >> 2;
    const int lane16 = 32 * (warp & 3) + 16 * ((warp >> 2) & 1);
    const uint32_t lb = static_cast<uint32_t>(lane16) << 16;
    const uint32_t t_s = tmem + lb + TMEM_S0 + wg * 128;
    const uint32_t t_o = tmem + lb + TMEM_O0 + wg * 128;
    const float sl2 = p.scale_log2;
    const int tail = p.n_rows - (nkv - 1) * BN;    // valid keys in the last tile (1..128)
    const int row_a = q_row0 + wg * BM + lane16 + t1;
    const int row_b = row_a + 8;
    float m_a = -INFINITY, m_b = -INFINITY;        // log2 units, identical in a row's 4 threads
    float l_a = 0.f, l_b = 0.f;                    // this thread's share of the row sums
    bool ok = true;
    constexpr float PART_LIMIT = 4611686018427387904.0f;   // 2^62: four shares stay below 2^64

    auto quad_max = [](float v) {
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    };
    auto quad_or = [](bool v) {
      int x = v ? 1 : 0;
      x |= __shfl_xor_sync(0xffffffffu, x, 1);
      x |= __shfl_xor_sync(0xffffffffu, x, 2);
      return x != 0;
    };
    // logits of 64 keys starting at key c0 of the tile (registers as loaded);
    // keys past the end -> -inf
    auto to_logits = [&](const uint32_t (&r)[32], int c0, bool last, float (&x)[32]) {
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]);
      if (last && tail < BN) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int key = c0 + 8 * (e >> 2) + 2 * t0 + (e & 1);
          if (key >= tail) x[e] = -INFINITY;
        }
      }
    };
    // numerators of the 16 keys of each row: bf16 pairs (register order of the
    // 16x128b store) and this thread's sums
    auto exps = [&](const float (&x)[32], uint32_t (&pk)[16], float& sa, float& sb) {
      const float2 c2 = make_float2(sl2, sl2);
      const float2 ma = make_float2(-m_a, -m_a), mb = make_float2(-m_b, -m_b);
      float2 acc_a = make_float2(0.f, 0.f), acc_b = make_float2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float2 ya = __ffma2_rn(make_float2(x[4 * q], x[4 * q + 1]), c2, ma);
        const float2 yb = __ffma2_rn(make_float2(x[4 * q + 2], x[4 * q + 3]), c2, mb);
        const float pa0 = ex2_approx(ya.x), pa1 = ex2_approx(ya.y);
        const float pb0 = ex2_approx(yb.x), pb1 = ex2_approx(yb.y);
        acc_a = __fadd2_rn(acc_a, make_float2(pa0, pa1));
        acc_b = __fadd2_rn(acc_b, make_float2(pb0, pb1));
        pk[2 * q] = pack_bf16x2(pa0, pa1);
        pk[2 * q + 1] = pack_bf16x2(pb0, pb1);
      }
      sa = acc_a.x + acc_a.y;
      sb = acc_b.x + acc_b.y;
    };
    // O *= f per row for this warp's lanes (warp-collective TMEM round trip)
    auto rescale_o = [&](float fa, float fb) {
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
        tmem_ld16x256(t_o + 64 * h, o);
        tmem_wait_ld(o);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          o[e] = __float_as_uint(__uint_as_float(o[e]) * (((e >> 1) & 1) ? fb : fa));
        tmem_st16x256(t_o + 64 * h, o);
      }
    };
    // the rare path: raise the reference of the rows whose shares need it
    // (all rows on the first half of the first tile); returns (fa, fb)
    auto new_reference = [&](const float (&x)[32], bool first, float sa, float sb, float& fa, float& fb) {
      const bool na = quad_or(first || !(sa <= PART_LIMIT));
      const bool nb = quad_or(first || !(sb <= PART_LIMIT));
      float xa = -INFINITY, xb = -INFINITY;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        xa = fmaxf(xa, fmaxf(x[4 * q], x[4 * q + 1]));
        xb = fmaxf(xb, fmaxf(x[4 * q + 2], x[4 * q + 3]));
      }
      xa = quad_max(xa);
      xb = quad_max(xb);
      fa = 1.f;
      fb = 1.f;
      if (na) {
        const float mn = fmaxf(m_a, xa * sl2);
        fa = first ? 0.f : ex2_approx(m_a - mn);
        m_a = mn;
        l_a *= fa;
      }
      if (nb) {
        const float mn = fmaxf(m_b, xb * sl2);
        fb = first ? 0.f : ex2_approx(m_b - mn);
        m_b = mn;
        l_b *= fb;
      }
    };
    // Publish 64 keys of P (32 TMEM columns at c0 / 2, aliasing S columns
    // already read): every lane's store lands and is fenced, then one arrival.
    auto store_p = [&](int half, const uint32_t (&pk)[16]) {
      __syncwarp();
      tmem_st16x128(t_s + 32 * half, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full(wg, half));
    };

    // Fused RoPE: rotate this tile's Q rows in shared memory, two threads per
    // row (each 8 of the 16 chunks), with the (cos, sin) the rope kernel uses
    // (read from the table) and its rot2 arithmetic, then make the
    // generic-proxy writes visible to the tensor core (async proxy).
    if (fused_rope) {
      if (!warp_wait(bar_q_full(wg), 0, abort_flag, limit, eslot)) ok = false;
      const int tid = (warp & 7) * 32 + lane;
      const int row_in_tile = tid >> 1, part = tid & 1;
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
          for (int c = 8 * part; c < 8 * part + 8; ++c) {   // pairs 4c .. 4c+3
            const float4 a = __ldg(cs4 + 2 * c), b = __ldg(cs4 + 2 * c + 1);
            const float2 cs[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y),
                                  make_float2(b.z, b.w)};
            *chunk(c) = rotate_adjacent(*chunk(c), cs);
          }
        } else {
#pragma unroll 2
          for (int c = 4 * part; c < 4 * part + 4; ++c) {   // pairs 8c .. 8c+7
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
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_q_ready(wg));
    }

    for (int j = 0; ok && j < nkv; ++j) {
      if (!warp_wait(bar_s_full(wg), j & 1, abort_flag, limit, eslot)) { ok = false; break; }
      tc_fence_after();
      const bool last = j == nkv - 1;
      {
        // ---- keys 0..63 ----
        uint32_t r[32];
        tmem_ld16x256(t_s, r);
        tmem_wait_ld(r);
        float x[32];
        to_logits(r, 0, last, x);
        uint32_t pk[16];
        float sa, sb;
        exps(x, pk, sa, sb);                        // speculative against the references
        const bool need = (j == 0) || !(sa <= PART_LIMIT) || !(sb <= PART_LIMIT);
        if (__any_sync(0xffffffffu, need)) {
          float fa, fb;
          new_reference(x, j == 0, sa, sb, fa, fb);
          __syncwarp();
          if (j > 0) rescale_o(fa, fb);   // O holds PV(j-1); PV(j) has not started
          exps(x, pk, sa, sb);
        }
        l_a += sa;
        l_b += sb;
        store_p(0, pk);
      }
      {
        // ---- keys 64..127 ----
        uint32_t r[32];
        __syncwarp();
        tmem_ld16x256(t_s + 64, r);
        tmem_wait_ld(r);
        float x[32];
        to_logits(r, 64, last, x);
        uint32_t pk[16];
        float sa, sb;
        exps(x, pk, sa, sb);
        const bool need = !(sa <= PART_LIMIT) || !(sb <= PART_LIMIT);
        if (__any_sync(0xffffffffu, need)) {
          // the first half of PV(j) may be in flight: let it land, then rescale
          // O (which now includes it) together with the running sums
          if (!warp_wait(bar_pva_done(wg), j & 1, abort_flag, limit, eslot)) { ok = false; break; }
          tc_fence_after();
          float fa, fb;
          new_reference(x, false, sa, sb, fa, fb);
          __syncwarp();
          rescale_o(fa, fb);
          exps(x, pk, sa, sb);
        }
        l_a += sa;
        l_b += sb;
        store_p(1, pk);
      }
    }

    // epilogue: O / l -> bf16 -> global; optional log-sum-exp
    if (ok && warp_wait(bar_o_full(wg), 0, abort_flag, limit, eslot)) {
      tc_fence_after();
      // row sums over the four threads of each row
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      const float inv_a = 1.f / l_a, inv_b = 1.f / l_b;
      __nv_bfloat16* orow_a = p.o + batch * p.o_batch_stride + static_cast<long long>(row_a) * p.o_row_stride + head * HD;
      __nv_bfloat16* orow_b = orow_a + 8 * p.o_row_stride;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
        __syncwarp();
        tmem_ld16x256(t_o + 64 * h, o);
        tmem_wait_ld(o);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int col = 64 * h + 8 * q + 2 * t0;
          if (row_a < p.n_rows)
            *reinterpret_cast<uint32_t*>(orow_a + col) =
                pack_bf16x2(__uint_as_float(o[4 * q]) * inv_a, __uint_as_float(o[4 * q + 1]) * inv_a);
          if (row_b < p.n_rows)
            *reinterpret_cast<uint32_t*>(orow_b + col) =
                pack_bf16x2(__uint_as_float(o[4 * q + 2]) * inv_b, __uint_as_float(o[4 * q + 3]) * inv_b);
        }
      }
      if (p.lse != nullptr && t0 == 0) {
        float* lrow = p.lse + (static_cast<long long>(batch) * p.n_heads + head) * p.n_rows;
        if (row_a < p.n_rows) lrow[row_a] = (m_a + __log2f(l_a)) * 0.69314718055994530942f;
        if (row_b < p.n_rows) lrow[row_b] = (m_b + __log2f(l_b)) * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn
}  // namespace h3
