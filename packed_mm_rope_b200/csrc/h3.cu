// h3.cu -- the C ABI of libh3 (declared in include/h3.h).
//
// Host-side argument validation, TMA tensor-map encoding and kernel launches.
// The library calls no device allocator: its device memory is static
// __device__ data of this module (the per-stream error words and the fixed
// scratch array of the allocation-free host call), and the host-buffer
// pipeline keeps two streams and a set of events per device.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "coords.cuh"
#include "rope.cuh"
#include "attention.cuh"
#include "adaln.cuh"

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr uint64_t kDrainLimitNs = 2000000000ull;
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// One-time set-up of the current device, kept until h3_shutdown: the
// shared-memory opt-ins of the kernels that need more than 48 KB (function
// attributes are per device) and the SM count.
struct DeviceState {
  bool ready = false;
  int sms = 148;
};

std::mutex g_state_mu;
DeviceState g_states[64];

const DeviceState* device_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_state_mu);
  DeviceState& st = g_states[dev];
  if (!st.ready) {
    if (cudaFuncSetAttribute(h3::attn::attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(h3::attn::SMEM_BYTES)) != cudaSuccess)
      return nullptr;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) st.sms = n;
    st.ready = true;
  }
  return &st;
}

int sm_count() {
  const DeviceState* st = device_state();
  return st ? st->sms : 148;
}

// Error-word slot of (current device, stream).  Slots 1 .. ERR_SLOTS-1 are
// handed out to streams in the order they are first seen; once they are used
// up, further streams share slot 0.  A stream destroyed and re-created at the
// same address keeps its slot.  Forgotten by h3_shutdown.
std::mutex g_slot_mu;
void* g_slot_stream[64][h3::ERR_SLOTS];
int g_slots_used[64];

int error_slot(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(g_slot_mu);
  for (int i = 1; i <= g_slots_used[dev]; ++i)
    if (g_slot_stream[dev][i] == stream) return i;
  if (g_slots_used[dev] + 1 >= h3::ERR_SLOTS) return 0;
  const int i = ++g_slots_used[dev];
  g_slot_stream[dev][i] = stream;
  return i;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a bf16 [batch][n_rows][row_stride] tensor whose first
// n_heads*128 columns are used; box = 64 columns x box_rows rows, 128-byte
// swizzle.
bool make_qkv_map(CUtensorMap* map, const void* ptr, int32_t batch, int64_t n_rows, int32_t n_heads,
                  int64_t row_stride, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(n_heads) * 128u, static_cast<cuuint64_t>(n_rows),
                              static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride) * 2u,
                                 static_cast<cuuint64_t>(row_stride) * 2u * static_cast<cuuint64_t>(n_rows)};
  const cuuint32_t box[3] = {64u, box_rows, 1u};
  const cuuint32_t estride[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                  estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool valid_rope_cfg(const h3_rope_cfg* cfg) {
  if (cfg == nullptr) return false;
  if (!(cfg->theta > 1.0) || !std::isfinite(cfg->theta)) return false;
  if (cfg->sec_t < 0 || cfg->sec_h < 0 || cfg->sec_w < 0) return false;
  if ((cfg->sec_t | cfg->sec_h | cfg->sec_w) & 1) return false;
  if (cfg->sec_t + cfg->sec_h + cfg->sec_w != cfg->head_dim) return false;
  if (cfg->pair_layout != 0 && cfg->pair_layout != 1) return false;
  if (cfg->freq_rule != 0 && cfg->freq_rule != 1) return false;
  return true;
}

h3::RopeTable make_rope_table(const h3_rope_cfg* cfg) {
  h3::RopeTable t;
  const int sec[3] = {cfg->sec_t, cfg->sec_h, cfg->sec_w};
  int p = 0;
  for (int a = 0; a < 3; ++a)
    for (int j = 0; j < sec[a] / 2; ++j, ++p) {
      // per-axis ladder (rule 0) or one ladder over the head's pairs (rule 1)
      t.inv_freq[p] = cfg->freq_rule == 0 ? std::pow(cfg->theta, -2.0 * j / sec[a])
                                          : std::pow(cfg->theta, -2.0 * p / cfg->head_dim);
      t.axis[p] = a;
    }
  return t;
}

// Checks a segment table against n_rows and packs it for the coordinate
// kernel; nothing is launched.  Every host-buffer call runs this before it
// queues any work, so a bad table never leaves copies in flight.
h3_status make_coord_table(const h3_segment* segs, int32_t nseg, int64_t n_rows, h3::CoordTable* tab) {
  if (segs == nullptr || nseg < 1 || nseg > H3_MAX_SEGMENTS || n_rows < 0) return H3_ERR_INVALID_ARG;
  static_assert(sizeof(h3::CoordTable) <= 4000, "segment table must fit in kernel parameters");
  std::memset(tab, 0, sizeof(*tab));
  tab->nseg = nseg;
  long long first = 0;
  constexpr long long kExact = 1ll << 24;   // integers below this are exact in fp32
  for (int i = 0; i < nseg; ++i) {
    const h3_segment& s = segs[i];
    if (s.count < 0 || s.t_den <= 0 || s.t_den >= kExact) return H3_ERR_INVALID_ARG;
    long long rows = 0;
    if (s.kind == H3_SEG_TEXT) {
      if (s.flags & ~H3_FLAG_TEXT_T_ONLY) return H3_ERR_INVALID_ARG;
      rows = s.count;
    } else if (s.kind == H3_SEG_VIDEO) {
      if (s.flags & ~H3_FLAG_VIDEO_CANVAS) return H3_ERR_INVALID_ARG;
      if (s.grid_h <= 0 || s.grid_w <= 0 || s.grid_h >= kExact || s.grid_w >= kExact)
        return H3_ERR_INVALID_ARG;
      rows = static_cast<long long>(s.count) * s.grid_h * s.grid_w;
    } else if (s.kind == H3_SEG_AUDIO) {
      if (s.flags & ~H3_FLAG_AUDIO_CHANNEL_H) return H3_ERR_INVALID_ARG;
      if (s.channels < 1 || s.channels > 2) return H3_ERR_INVALID_ARG;
      rows = static_cast<long long>(s.count) * s.channels;
    } else {
      return H3_ERR_INVALID_ARG;
    }
    if (s.count > 0) {   // t is linear in the index: check both ends
      const long long t0 = s.t_off_num;
      const long long t1 = s.t_off_num + static_cast<long long>(s.count - 1) * s.t_step_num;
      if (t0 <= -kExact || t0 >= kExact || t1 <= -kExact || t1 >= kExact) return H3_ERR_INVALID_ARG;
    }
    tab->seg[i] = s;
    tab->first[i] = first;
    first += rows;
    if (first > (1ll << 40)) return H3_ERR_INVALID_ARG;
  }
  tab->first[nseg] = first;
  return first == n_rows ? H3_OK : H3_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

const char* h3_status_str(int32_t status) {
  switch (status) {
    case H3_OK: return "ok";
    case H3_ERR_INVALID_ARG: return "invalid argument";
    case H3_ERR_UNSUPPORTED: return "unsupported argument";
    case H3_ERR_CUDA: return "CUDA error";
    case H3_ERR_TIMEOUT: return "bounded device wait expired";
    case H3_ERR_DEVICE_INPUT: return "kernel found an invalid input";
    case H3_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of the no-allocation call";
    default: return "unknown status";
  }
}

int32_t h3_version(void) { return 101; }

h3_status h3_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : ns);
  return H3_OK;
}

h3_status h3_build_coords(const h3_segment* segs, int32_t nseg, const int32_t* d_perm, int64_t n_rows,
                          float* d_coords, void* stream) {
  h3::CoordTable tab;
  const h3_status st = make_coord_table(segs, nseg, n_rows, &tab);
  if (st != H3_OK) return st;
  if (n_rows == 0) return H3_OK;
  if (d_coords == nullptr) return H3_ERR_INVALID_ARG;
  const int threads = 256;
  const long long blocks_needed = (n_rows + threads - 1) / threads;
  const int blocks = static_cast<int>(blocks_needed < 8LL * sm_count() ? blocks_needed : 8LL * sm_count());
  h3::coords_kernel<<<blocks, threads, 0, as_stream(stream)>>>(tab, d_perm, n_rows, d_coords,
                                                               error_slot(stream));
  return cudaGetLastError() == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}

h3_status h3_mmrope_qk(const void* d_q, const void* d_k, void* d_q_out, void* d_k_out,
                       const float* d_coords, int64_t n_rows, int32_t n_heads, int64_t row_stride,
                       const h3_rope_cfg* cfg, void* stream) {
  if (n_rows < 0 || n_heads < 1 || !valid_rope_cfg(cfg)) return H3_ERR_INVALID_ARG;
  if (cfg->head_dim != 128) return H3_ERR_UNSUPPORTED;
  if (row_stride < static_cast<int64_t>(n_heads) * 128) return H3_ERR_INVALID_ARG;
  if (n_rows == 0) return H3_OK;
  if ((d_q == nullptr) != (d_q_out == nullptr)) return H3_ERR_INVALID_ARG;   // both or neither
  if (!d_k || !d_k_out || !d_coords) return H3_ERR_INVALID_ARG;
  if (row_stride % 8 != 0 || !aligned16(d_q) || !aligned16(d_k) || !aligned16(d_q_out) ||
      !aligned16(d_k_out))
    return H3_ERR_UNSUPPORTED;
  if (static_cast<long long>(n_heads) * 16 > (1ll << 30)) return H3_ERR_INVALID_ARG;
  const h3::RopeTable tab = make_rope_table(cfg);
  // one warp per row; four CTAs per SM queued for two resident (tail balance)
  const long long warps_per_cta = h3::ROPE_THREADS / 32;
  const long long nblk = (n_rows + warps_per_cta - 1) / warps_per_cta;
  const long long cap = 2LL * h3::ROPE_CTAS_PER_SM * sm_count();
  const int grid = static_cast<int>(nblk < cap ? nblk : cap);
  const long long stride16 = row_stride / 8;
  auto q = static_cast<const uint4*>(d_q);
  auto k = static_cast<const uint4*>(d_k);
  auto qo = static_cast<uint4*>(d_q_out);
  auto ko = static_cast<uint4*>(d_k_out);
  if (cfg->pair_layout == 0)
    h3::rope_kernel<0><<<grid, h3::ROPE_THREADS, 0, as_stream(stream)>>>(q, k, qo, ko, d_coords, n_rows,
                                                                       n_heads, stride16, tab);
  else
    h3::rope_kernel<1><<<grid, h3::ROPE_THREADS, 0, as_stream(stream)>>>(q, k, qo, ko, d_coords, n_rows,
                                                                       n_heads, stride16, tab);
  return cudaGetLastError() == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}

h3_status h3_rope_cos_sin(const float* d_coords, int64_t n_rows, const h3_rope_cfg* cfg, float* d_cs,
                          void* stream) {
  if (n_rows < 0 || !valid_rope_cfg(cfg)) return H3_ERR_INVALID_ARG;
  if (cfg->head_dim != 128) return H3_ERR_UNSUPPORTED;
  if (n_rows == 0) return H3_OK;
  if (!d_coords || !d_cs) return H3_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_cs) & 15u) != 0) return H3_ERR_UNSUPPORTED;
  if (n_rows > (1ll << 40)) return H3_ERR_INVALID_ARG;
  const h3::RopeTable tab = make_rope_table(cfg);
  const long long need = (n_rows * 64 + 255) / 256;
  const int grid = static_cast<int>(need < 16LL * sm_count() ? need : 16LL * sm_count());
  h3::rope_cos_sin_kernel<<<grid, 256, 0, as_stream(stream)>>>(d_coords, n_rows, reinterpret_cast<float2*>(d_cs),
                                                               tab);
  return cudaGetLastError() == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}

h3_status h3_packed_attention(const void* d_q, const void* d_k, const void* d_v, void* d_o, float* d_lse,
                              const float* d_rope_cs, const h3_rope_cfg* cfg, int32_t batch, int64_t n_rows,
                              int32_t n_heads, int32_t head_dim, int64_t row_stride, float softmax_scale,
                              void* stream) {
  if (batch < 1 || n_heads < 1 || n_rows < 0 || n_rows >= (1ll << 31)) return H3_ERR_INVALID_ARG;
  if (head_dim != 128) return H3_ERR_UNSUPPORTED;
  if (d_rope_cs != nullptr) {
    if (!valid_rope_cfg(cfg)) return H3_ERR_INVALID_ARG;
    if (cfg->head_dim != 128) return H3_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(d_rope_cs) & 15u) != 0) return H3_ERR_UNSUPPORTED;
  }
  if (row_stride < static_cast<int64_t>(n_heads) * 128) return H3_ERR_INVALID_ARG;
  if (batch > 65535 || n_heads > 65535) return H3_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return H3_ERR_INVALID_ARG;
  if (n_rows == 0) return H3_OK;
  if (!d_q || !d_k || !d_v || !d_o) return H3_ERR_INVALID_ARG;
  if (row_stride % 8 != 0 || !aligned16(d_q) || !aligned16(d_k) || !aligned16(d_v) || !aligned16(d_o))
    return H3_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  if (!make_qkv_map(&tq, d_q, batch, n_rows, n_heads, row_stride, 128) ||
      !make_qkv_map(&tk, d_k, batch, n_rows, n_heads, row_stride, 128) ||
      !make_qkv_map(&tv, d_v, batch, n_rows, n_heads, row_stride, 128))
    return H3_ERR_CUDA;
  if (device_state() == nullptr) return H3_ERR_CUDA;

  h3::attn::Params p;
  p.n_rows = static_cast<int>(n_rows);
  p.n_heads = n_heads;
  p.n_kv_tiles = static_cast<int>((n_rows + h3::attn::BN - 1) / h3::attn::BN);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(128.0f);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(d_o);
  p.o_row_stride = row_stride;
  p.o_batch_stride = row_stride * n_rows;
  p.lse = d_lse;
  p.wait_limit_ns = g_wait_limit_ns.load();
  p.drain_limit_ns = kDrainLimitNs;
  p.err_slot = error_slot(stream);
  p.rope_cs = reinterpret_cast<const float2*>(d_rope_cs);
  p.rope_layout = d_rope_cs ? cfg->pair_layout : 0;
  const dim3 grid(static_cast<unsigned>((n_rows + 2 * h3::attn::BM - 1) / (2 * h3::attn::BM)),
                  static_cast<unsigned>(n_heads), static_cast<unsigned>(batch));
  h3::attn::attention_kernel<<<grid, h3::attn::THREADS, h3::attn::SMEM_BYTES, as_stream(stream)>>>(tq, tk, tv,
                                                                                                  p);
  return cudaGetLastError() == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}

h3_status h3_adaln_modulate(const void* d_x, void* d_y, const int32_t* d_timestep_index,
                            const int32_t* d_token_tag, const float* d_table, int32_t n_entries, int64_t n_rows,
                            int32_t hidden, int64_t x_row_stride, int64_t y_row_stride, float eps, void* stream) {
  if (n_rows < 0 || hidden < 8 || n_entries < 1 || !(eps >= 0.f) || !std::isfinite(eps)) return H3_ERR_INVALID_ARG;
  if (hidden % 8 != 0 || hidden > h3::ADALN_MAX_HIDDEN) return H3_ERR_UNSUPPORTED;
  if (x_row_stride < hidden || y_row_stride < hidden) return H3_ERR_INVALID_ARG;
  if (n_rows == 0) return H3_OK;
  if (!d_x || !d_y || !d_timestep_index || !d_token_tag || !d_table) return H3_ERR_INVALID_ARG;
  if (x_row_stride % 8 || y_row_stride % 8 || !aligned16(d_x) || !aligned16(d_y) || !aligned16(d_table))
    return H3_ERR_UNSUPPORTED;
  // one resident wave: ADALN_CTAS_PER_SM CTAs per SM, rows grid-strided over the row groups
  const long long grid = std::min<long long>(static_cast<long long>(h3::ADALN_CTAS_PER_SM) * sm_count(),
                                             (n_rows + h3::ADALN_GROUPS - 1) / h3::ADALN_GROUPS);
  h3::adaln_kernel<<<static_cast<int>(grid), h3::ADALN_THREADS, 0, as_stream(stream)>>>(
      static_cast<const uint4*>(d_x), static_cast<uint4*>(d_y), d_timestep_index, d_token_tag,
      reinterpret_cast<const float4*>(d_table), n_entries, n_rows, hidden / 8, x_row_stride / 8, y_row_stride / 8,
      eps, error_slot(stream));
  return cudaGetLastError() == cudaSuccess ? H3_OK : H3_ERR_CUDA;
}

uint64_t h3_host_workspace_bytes(int64_t n_rows, int32_t n_heads) {
  if (n_rows <= 0 || n_heads < 1 || n_rows >= (1ll << 31)) return 0;
  auto up = [](uint64_t b) { return (b + 255u) & ~uint64_t(255u); };
  const uint64_t t = static_cast<uint64_t>(n_rows) * n_heads * 128u * 2u;
  return 4 * up(t) + up(static_cast<uint64_t>(n_rows) * 12u) + up(static_cast<uint64_t>(n_rows) * 4u);
}

}  // extern "C"

namespace {

// Streams and events of the host-buffer pipeline: created once per device,
// kept for the life of the process.
struct HostPipe {
  std::mutex enqueue;             // one caller at a time enqueues on a device
  cudaStream_t h2d = nullptr, d2h = nullptr;
  static constexpr int kMaxChunks = 64;
  static constexpr int kEvents = 2 * kMaxChunks + 2;   // per chunk: copied in, attended; start, end
  cudaEvent_t ev[kEvents] = {};
  bool ok = false;
};

std::mutex g_pipes_mu;
HostPipe g_pipes[64];

HostPipe* host_pipe() {
  std::mutex& mu = g_pipes_mu;
  HostPipe* pipes = g_pipes;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  HostPipe& hp = pipes[dev];
  if (!hp.ok) {
    bool made = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& e : hp.ev)
      made = made && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!made) {   // release whatever was created; the next call tries again
      for (auto& e : hp.ev)
        if (e != nullptr) cudaEventDestroy(e), e = nullptr;
      if (hp.h2d != nullptr) cudaStreamDestroy(hp.h2d);
      if (hp.d2h != nullptr) cudaStreamDestroy(hp.d2h);
      hp.h2d = hp.d2h = nullptr;
      return nullptr;
    }
    hp.ok = true;
  }
  return &hp;
}

// Waits for and destroys every device's pipeline streams and events; the next
// host-buffer call re-creates them.  Changes the current device.
void release_host_pipes() {
  std::lock_guard<std::mutex> lock(g_pipes_mu);
  for (int dev = 0; dev < 64; ++dev) {
    HostPipe& hp = g_pipes[dev];
    if (!hp.ok) continue;
    std::lock_guard<std::mutex> q(hp.enqueue);
    if (cudaSetDevice(dev) != cudaSuccess) continue;
    cudaStreamSynchronize(hp.h2d);
    cudaStreamSynchronize(hp.d2h);
    for (auto& e : hp.ev) {
      cudaEventDestroy(e);
      e = nullptr;
    }
    cudaStreamDestroy(hp.h2d);
    cudaStreamDestroy(hp.d2h);
    hp.h2d = hp.d2h = nullptr;
    hp.ok = false;
  }
}

// Heads per chunk such that one chunk's attention grid fills whole waves of
// SMs (one CTA per SM), preferring 4..8 heads; the last chunk may be shorter.
int pick_heads_per_chunk(int64_t n_rows, int n_heads) {
  const long long qtiles = (n_rows + 2 * h3::attn::BM - 1) / (2 * h3::attn::BM);
  const int sms = sm_count();
  int best = n_heads < 4 ? n_heads : 4;
  double best_waste = 2.0;
  for (int hc = 2; hc <= 8 && hc <= n_heads; ++hc) {
    const long long ctas = qtiles * hc;
    const double waves = static_cast<double>(ctas) / sms;
    const double waste = std::ceil(waves) / waves - 1.0;   // idle fraction of the last wave
    if (waste < best_waste - 1e-9) { best_waste = waste; best = hc; }
  }
  return best;
}

// Chunk sizes of the host pipeline: chunks of `hc` heads, and with `taper` the
// last hc + (n_heads mod hc) heads in halving pieces (6 -> 3, 2, 1), so that the
// attention and the copy out that remain after the last copy in are short.
int plan_chunks(int n_heads, int hc, bool taper, int (&sizes)[HostPipe::kMaxChunks]) {
  int n = 0, left = n_heads;
  const int tail = taper ? std::min(n_heads, hc + n_heads % hc) : 0;
  while (left > tail && n < HostPipe::kMaxChunks) {
    const int c = std::min(hc, left - tail);
    sizes[n++] = c;
    left -= c;
  }
  while (left > 0 && n < HostPipe::kMaxChunks) {
    const int c = (left + 1) / 2;
    sizes[n++] = c;
    left -= c;
  }
  return left == 0 ? n : -1;
}

}  // namespace

extern "C" {

h3_status h3_packed_mmrope_attention_host(const h3_segment* segs, int32_t nseg, const int32_t* h_perm,
                                          const void* h_q, const void* h_k, const void* h_v, void* h_o,
                                          void* d_work, int64_t n_rows, int32_t n_heads,
                                          int32_t heads_per_chunk, const h3_rope_cfg* cfg, void* stream) {
  // every argument is checked before anything is queued
  if (n_rows < 0 || n_heads < 1 || !valid_rope_cfg(cfg)) return H3_ERR_INVALID_ARG;
  if (cfg->head_dim != 128) return H3_ERR_UNSUPPORTED;
  if (heads_per_chunk < 0 || heads_per_chunk > n_heads) return H3_ERR_INVALID_ARG;
  h3::CoordTable tab;
  h3_status st = make_coord_table(segs, nseg, n_rows, &tab);
  if (st != H3_OK || n_rows == 0) return st;
  if (!h_q || !h_k || !h_v || !h_o) return H3_ERR_INVALID_ARG;
  if (n_rows >= (1ll << 31)) return H3_ERR_INVALID_ARG;
  if (d_work == nullptr || (reinterpret_cast<uintptr_t>(d_work) & 255u)) return H3_ERR_INVALID_ARG;
  const int hc = heads_per_chunk > 0 ? heads_per_chunk : pick_heads_per_chunk(n_rows, n_heads);
  int chunk_heads[HostPipe::kMaxChunks];
  const int nchunks = plan_chunks(n_heads, hc, heads_per_chunk == 0, chunk_heads);
  if (nchunks < 0) return H3_ERR_UNSUPPORTED;
  HostPipe* hp = host_pipe();
  if (hp == nullptr) return H3_ERR_CUDA;
  std::lock_guard<std::mutex> lock(hp->enqueue);
  cudaStream_t s = as_stream(stream);

  // carve the workspace
  auto up = [](uint64_t b) { return (b + 255u) & ~uint64_t(255u); };
  const uint64_t row_bytes = static_cast<uint64_t>(n_heads) * 256u;
  const uint64_t t = up(static_cast<uint64_t>(n_rows) * row_bytes);
  uint8_t* w = static_cast<uint8_t*>(d_work);
  uint8_t *dq = w, *dk = w + t, *dv = w + 2 * t, *d_o = w + 3 * t;
  float* dcoords = reinterpret_cast<float*>(w + 4 * t);
  int32_t* dperm = reinterpret_cast<int32_t*>(w + 4 * t + up(static_cast<uint64_t>(n_rows) * 12u));

  cudaEvent_t* ev_in = hp->ev;
  cudaEvent_t* ev_out = hp->ev + HostPipe::kMaxChunks;
  cudaEvent_t ev_start = hp->ev[2 * HostPipe::kMaxChunks], ev_end = hp->ev[2 * HostPipe::kMaxChunks + 1];
  auto ck = [](cudaError_t e) { return e == cudaSuccess; };
  // After a failure with copies already queued: order `stream` after both copy
  // streams, so that a caller who synchronises `stream` and then frees its
  // host buffers cannot race a copy still in flight.
  auto fail = [&](h3_status status) {
    if (ck(cudaEventRecord(ev_end, hp->h2d))) cudaStreamWaitEvent(s, ev_end, 0);
    if (ck(cudaEventRecord(ev_start, hp->d2h))) cudaStreamWaitEvent(s, ev_start, 0);
    return status;
  };

  // both copy streams start after the work already queued on `stream`
  if (!ck(cudaEventRecord(ev_start, s)) || !ck(cudaStreamWaitEvent(hp->h2d, ev_start, 0)) ||
      !ck(cudaStreamWaitEvent(hp->d2h, ev_start, 0)))
    return H3_ERR_CUDA;
  // coordinates (after the permutation is on the device)
  if (h_perm != nullptr) {
    if (!ck(cudaMemcpyAsync(dperm, h_perm, static_cast<size_t>(n_rows) * 4, cudaMemcpyHostToDevice, s)))
      return fail(H3_ERR_CUDA);
  }
  st = h3_build_coords(segs, nseg, h_perm ? dperm : nullptr, n_rows, dcoords, stream);
  if (st != H3_OK) return fail(st);

  for (int c = 0, h0 = 0; c < nchunks; h0 += chunk_heads[c], ++c) {
    const int nh = chunk_heads[c];
    const size_t off = static_cast<size_t>(h0) * 256u, width = static_cast<size_t>(nh) * 256u;
    for (int x = 0; x < 3; ++x) {
      const uint8_t* src = static_cast<const uint8_t*>(x == 0 ? h_q : x == 1 ? h_k : h_v) + off;
      uint8_t* dst = (x == 0 ? dq : x == 1 ? dk : dv) + off;
      if (!ck(cudaMemcpy2DAsync(dst, row_bytes, src, row_bytes, width, static_cast<size_t>(n_rows),
                                cudaMemcpyHostToDevice, hp->h2d)))
        return fail(H3_ERR_CUDA);
    }
    if (!ck(cudaEventRecord(ev_in[c], hp->h2d)) || !ck(cudaStreamWaitEvent(s, ev_in[c], 0)))
      return fail(H3_ERR_CUDA);
    // rotate this chunk's Q and K in place, then attend over all rows for its heads
    st = h3_mmrope_qk(dq + off, dk + off, dq + off, dk + off, dcoords, n_rows, nh,
                      static_cast<int64_t>(n_heads) * 128, cfg, stream);
    if (st != H3_OK) return fail(st);
    st = h3_packed_attention(dq + off, dk + off, dv + off, d_o + off, nullptr, nullptr, nullptr, 1, n_rows, nh, 128,
                             static_cast<int64_t>(n_heads) * 128, 0.f, stream);
    if (st != H3_OK) return fail(st);
    if (!ck(cudaEventRecord(ev_out[c], s)) || !ck(cudaStreamWaitEvent(hp->d2h, ev_out[c], 0)))
      return fail(H3_ERR_CUDA);
    if (!ck(cudaMemcpy2DAsync(static_cast<uint8_t*>(h_o) + off, row_bytes, d_o + off, row_bytes, width,
                              static_cast<size_t>(n_rows), cudaMemcpyDeviceToHost, hp->d2h)))
      return fail(H3_ERR_CUDA);
  }
  // `stream` is ordered after the last copy out (and, through it, all others)
  if (!ck(cudaEventRecord(ev_end, hp->d2h)) || !ck(cudaStreamWaitEvent(s, ev_end, 0))) return fail(H3_ERR_CUDA);
  return H3_OK;
}

}  // extern "C"

// ---- allocation-free variant of the host-buffer call ----------------------
//
// Its workspace is this file-scope device array instead of caller memory.  In
// host code the name is only a host-side stand-in for the device symbol: its
// device address must be looked up with cudaGetSymbolAddress (once per device,
// with that device current) and that address passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[H3_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64];

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call per device and cached until h3_shutdown), or null if the lookup
// fails.  A device reset moves the array, hence h3_shutdown before any reset.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

h3_status h3_packed_mmrope_attention_host_noalloc(const h3_segment* segs, int32_t nseg, const int32_t* h_perm,
                                                  const void* h_q, const void* h_k, const void* h_v, void* h_o,
                                                  int64_t n_rows, int32_t n_heads, const h3_rope_cfg* cfg,
                                                  void* stream) {
  // every argument is checked before anything is queued
  if (n_rows < 0 || n_heads < 1 || !valid_rope_cfg(cfg)) return H3_ERR_INVALID_ARG;
  if (cfg->head_dim != 128) return H3_ERR_UNSUPPORTED;
  h3::CoordTable tab;
  const h3_status tst = make_coord_table(segs, nseg, n_rows, &tab);
  if (tst != H3_OK || n_rows == 0) return tst;
  if (!h_q || !h_k || !h_v || !h_o) return H3_ERR_INVALID_ARG;
  const uint64_t need = h3_host_workspace_bytes(n_rows, n_heads);
  if (need == 0) return H3_ERR_INVALID_ARG;
  if (need > H3_NOALLOC_SCRATCH_BYTES) return H3_ERR_TOO_LARGE;
  uint8_t* w = static_cast<uint8_t*>(noalloc_scratch());
  if (w == nullptr) return H3_ERR_CUDA;

  // same carving as the workspace variant
  auto up = [](uint64_t b) { return (b + 255u) & ~uint64_t(255u); };
  const uint64_t bytes = static_cast<uint64_t>(n_rows) * n_heads * 256u;
  const uint64_t t = up(bytes);
  uint8_t *dq = w, *dk = w + t, *dv = w + 2 * t, *d_o = w + 3 * t;
  float* dcoords = reinterpret_cast<float*>(w + 4 * t);
  int32_t* dperm = reinterpret_cast<int32_t*>(w + 4 * t + up(static_cast<uint64_t>(n_rows) * 12u));
  cudaStream_t s = as_stream(stream);
  const int64_t rs = static_cast<int64_t>(n_heads) * 128;

  // everything in order on `stream`: copies in, coords, rope, attention, copy out
  if (h_perm != nullptr &&
      cudaMemcpyAsync(dperm, h_perm, static_cast<size_t>(n_rows) * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return H3_ERR_CUDA;
  if (cudaMemcpyAsync(dq, h_q, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, h_k, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, h_v, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return H3_ERR_CUDA;
  h3_status st = h3_build_coords(segs, nseg, h_perm ? dperm : nullptr, n_rows, dcoords, stream);
  if (st != H3_OK) return st;
  st = h3_mmrope_qk(dq, dk, dq, dk, dcoords, n_rows, n_heads, rs, cfg, stream);
  if (st != H3_OK) return st;
  st = h3_packed_attention(dq, dk, dv, d_o, nullptr, nullptr, nullptr, 1, n_rows, n_heads, 128, rs, 0.f, stream);
  if (st != H3_OK) return st;
  if (cudaMemcpyAsync(h_o, d_o, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return H3_ERR_CUDA;
  return H3_OK;
}

h3_status h3_check_device_error(void* stream) {
  // this stream's word, taken by a kernel ordered after the work already on it
  const int slot = error_slot(stream);
  h3::take_error_word<<<1, 1, 0, as_stream(stream)>>>(slot);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(as_stream(stream)) != cudaSuccess)
    return H3_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, h3::g_error_snapshot, sizeof(word), sizeof(word) * slot) != cudaSuccess)
    return H3_ERR_CUDA;
  if (word & h3::DEVERR_TIMEOUT) return H3_ERR_TIMEOUT;
  if (word & h3::DEVERR_INPUT) return H3_ERR_DEVICE_INPUT;
  return H3_OK;
}

}  // extern "C"

// ---- lifecycle ------------------------------------------------------------

namespace {

// Restores the calling thread's current device on scope exit.
struct DeviceGuard {
  int saved = -1;
  DeviceGuard() { if (cudaGetDevice(&saved) != cudaSuccess) saved = -1; }
  ~DeviceGuard() { if (saved >= 0) cudaSetDevice(saved); }
};

}  // namespace

extern "C" {

h3_status h3_init(int32_t device) {
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess) return H3_ERR_CUDA;
  if (device < 0 || device >= count || device >= 64) return H3_ERR_INVALID_ARG;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return H3_ERR_CUDA;
  if (major != 10 || minor != 0) return H3_ERR_UNSUPPORTED;   // the kernels are built for sm_100a only
  DeviceGuard guard;
  if (cudaSetDevice(device) != cudaSuccess) return H3_ERR_CUDA;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, h3::attn::attention_kernel) != cudaSuccess) return H3_ERR_UNSUPPORTED;
  if (encode_tiled() == nullptr || device_state() == nullptr || host_pipe() == nullptr ||
      noalloc_scratch() == nullptr)
    return H3_ERR_CUDA;
  static const unsigned int zeros[h3::ERR_SLOTS] = {};
  if (cudaMemcpyToSymbol(h3::g_error_words, zeros, sizeof(zeros)) != cudaSuccess) return H3_ERR_CUDA;
  return H3_OK;
}

void h3_shutdown(void) {
  DeviceGuard guard;
  release_host_pipes();
  // per-device lookups and set-up are redone by the next call (after a device
  // reset the module, its kernels' attributes and its arrays are new)
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    for (auto& a : g_scratch_addr) a = nullptr;
  }
  {
    std::lock_guard<std::mutex> lock(g_state_mu);
    for (auto& st : g_states) st = DeviceState();
  }
  {
    std::lock_guard<std::mutex> lock(g_slot_mu);
    for (auto& n : g_slots_used) n = 0;
  }
}

}  // extern "C"
