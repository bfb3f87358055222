/*
 * h3.h -- C ABI of libh3: packed multimodal MM-RoPE attention on B200 (sm_100a).
 *
 * The library computes the attention hot path of a single-stream audio-video
 * diffusion transformer: text, reference, video-latent and stereo-audio rows
 * are packed into ONE sequence, every row carries a three-axis (t, h, w)
 * position, Q and K are rotated by a three-axis rotary embedding, and every
 * row attends to every row.
 *
 * Sources (page titles as published):
 *   [P1] "Inside MiniMax H3: One DiT Stream for Text, Video, and Stereo Audio",
 *        section 2 (one packed sequence, shared projections), section 4
 *        (three-axis RoPE on a shared physical timeline; row order carries no
 *        position), section 6 (full attention dominates the cost).
 *   [P3] "MiniMax H3 -- one transformer that denoises video and audio
 *        together": latent-frame passage (880 tokens of one latent frame share
 *        t), clock-unit passage (1 unit = 1/40 s, 5/3 units per 24 fps frame),
 *        text passage (text t = index), rope-config passage (inverse
 *        frequencies computed from rope_theta / rope_freq_dim), and the
 *        bidirectional-attention passage.
 *   [P5] "MiniMax H3 -- Open-Weights Omni-Reference Video-Audio Generation
 *        Model Card", section H3-Omni-Transformer (3-D MM-RoPE over (t,h,w)).
 *
 * Conventions for every call:
 *   - Pointers named d_* are DEVICE pointers owned by the caller; the library
 *     never frees or retains them after the call returns.  Host pointers are
 *     read during the call only.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Arguments are validated on the host
 *     before anything is launched; a call that returns an error launched
 *     nothing, except H3_ERR_CUDA reported by the launch itself.
 *   - The library allocates no device memory at run time.  Its only device
 *     storage is static module data, held by every GPU that loads the
 *     library until the process exits: 2 KB of error words and the fixed
 *     H3_NOALLOC_SCRATCH_BYTES (64 MiB) scratch array of
 *     h3_packed_mmrope_attention_host_noalloc.
 *   - Kernel-side faults in the inputs (a permutation entry out of range, a
 *     bounded wait that expired) are recorded in an error word of the stream
 *     the kernel ran on; h3_check_device_error(stream) reads and clears it.
 *   - Host calls are thread-safe for distinct streams.
 *   - Q/K/V/O tensors are bf16 in row-major [batch][n_rows][n_heads][head_dim]
 *     with a row stride of `row_stride` elements (>= n_heads * head_dim,
 *     a multiple of 8) and a batch stride of n_rows * row_stride elements.
 *     Base pointers must be 16-byte aligned.  This is the natural layout of a
 *     fused QKV projection output (hidden 5376 = 42 heads x 128).
 */
#ifndef H3_H_
#define H3_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  H3_OK = 0,
  H3_ERR_INVALID_ARG = 1,   /* bad size, count, table or pointer */
  H3_ERR_UNSUPPORTED = 2,   /* valid but not implemented (head_dim != 128, misalignment, ...) */
  H3_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  H3_ERR_TIMEOUT = 4,       /* a bounded device-side wait expired (see h3_set_wait_limit_ns) */
  H3_ERR_DEVICE_INPUT = 5,  /* a kernel found a bad input (e.g. perm entry out of range) */
  H3_ERR_TOO_LARGE = 6      /* problem needs more than the fixed scratch of the no-allocation call */
} h3_status;

/* Segment kinds. */
enum { H3_SEG_TEXT = 0, H3_SEG_VIDEO = 1, H3_SEG_AUDIO = 2 };

/* Segment flags (bit set). */
enum {
  H3_FLAG_TEXT_T_ONLY = 1,       /* text at (t, 0, 0) instead of (t, t, t) */
  H3_FLAG_AUDIO_CHANNEL_H = 2,   /* stereo channel on the h axis instead of w */
  H3_FLAG_VIDEO_CANVAS = 4       /* video (h, w) on the normalised spatial canvas (below) */
};

/*
 * One contiguous run of logical elements of one modality ([P1] section 4;
 * [P3] latent-frame, text and clock passages).
 *
 * Logical element order: segments in table order; inside a text segment the
 * token index i; inside a video segment (frame k, y, x) row-major over a
 * grid_h x grid_w patch grid; inside an audio segment (token j, channel c).
 *
 * Time of element index idx (i, k or j) is the exact rational
 *     t = (t_off_num + idx * t_step_num) / t_den
 * in clock units of one audio latent (1/40 s).  A 4x-temporal latent video
 * frame advances 20/3 units (t_step_num = 20, t_den = 3); audio advances 1.
 * Coordinates produced (t, h, w):
 *     text  : (t, t, t), or (t, 0, 0) with H3_FLAG_TEXT_T_ONLY
 *     video : (t, y, x), or with H3_FLAG_VIDEO_CANVAS
 *             (t, c(y, grid_h), c(x, grid_w)) where
 *             c(i, n) = 16 + (i + 1/2 - n/2) * 32 / sqrt(grid_h * grid_w):
 *             the grid normalised by sqrt(height x width) and centred on
 *             [0, 32) ([P3] resolution passage), evaluated in fp64 one IEEE
 *             operation at a time and rounded to fp32
 *     audio : (t, 0, c), or (t, c, 0) with H3_FLAG_AUDIO_CHANNEL_H
 * Exactness: |t_off_num + idx * t_step_num| < 2^24 and 0 < t_den < 2^24 for
 * every idx; then the fp32 value is the correctly rounded quotient.
 */
typedef struct {
  int32_t kind;        /* H3_SEG_TEXT / H3_SEG_VIDEO / H3_SEG_AUDIO */
  int32_t count;       /* text tokens / latent frames / audio tokens (>= 0) */
  int32_t grid_h;      /* video: patch-grid height (> 0) */
  int32_t grid_w;      /* video: patch-grid width  (> 0) */
  int32_t channels;    /* audio: channels (1 or 2) */
  int32_t t_off_num;
  int32_t t_step_num;
  int32_t t_den;       /* > 0 */
  int32_t flags;       /* H3_FLAG_* */
} h3_segment;

#define H3_MAX_SEGMENTS 64

/*
 * Rotary configuration ([P3] rope-config passage; [P5] H3-Omni-Transformer).
 * The head dimension is split into per-axis sections sec_t + sec_h + sec_w
 * == head_dim (each even); pairs [0, sec_t/2) are driven by t, the next
 * sec_h/2 by h, the last sec_w/2 by w.
 * freq_rule 0 (default): axis a with D_a dims restarts the frequency ladder,
 *   its j-th pair has inverse frequency theta^(-2j / D_a).
 * freq_rule 1: one ladder over the whole head, pair p (counted over the head)
 *   has theta^(-2p / head_dim).  The pages name a rope frequency dimension
 *   without a formula; these are its two plain readings.
 * Frequencies are computed in fp64 on the host.
 * pair_layout 0: pair p = dims (2p, 2p+1).  pair_layout 1: pair p = dims
 * (p, p + head_dim/2).
 * A pair (x0, x1) at angle a becomes (x0 cos a - x1 sin a, x0 sin a + x1 cos a).
 */
typedef struct {
  double theta;        /* rotary base, > 1 (10000) */
  int32_t head_dim;    /* must be 128 */
  int32_t sec_t;       /* 32 */
  int32_t sec_h;       /* 48 */
  int32_t sec_w;       /* 48 */
  int32_t pair_layout; /* 0 (adjacent, default) or 1 (half-split) */
  int32_t freq_rule;   /* 0 (per-axis ladders, default) or 1 (one ladder) */
} h3_rope_cfg;

/* Short English text for a status code (static storage; never NULL). */
const char* h3_status_str(int32_t status);

/* Library ABI version (major * 100 + minor). */
int32_t h3_version(void);

/*
 * h3_init -- optional up-front set-up of one device.  The pages define no
 * counterpart; it is plumbing.  Checks that `device` exists and has compute
 * capability 10.0 (the kernels are built for sm_100a only) and that the
 * kernels load on it, then does once what every other call otherwise does
 * lazily on first use: the shared-memory opt-ins of the kernels, the lookup of
 * the driver's tensor-map encoder, the host-buffer pipeline's two streams and
 * events, the address of the no-allocation scratch; and clears the device's
 * error words.  Allocates no device memory at run time (loading the kernels
 * on the device commits the module's static arrays, among them the 64 MiB
 * no-allocation scratch).  The calling thread's current device is left as it
 * was.  Calling it again is harmless.
 * Errors: H3_ERR_INVALID_ARG (no such device), H3_ERR_UNSUPPORTED (another
 * architecture, or the kernels do not load), H3_ERR_CUDA.
 */
h3_status h3_init(int32_t device);

/*
 * h3_shutdown -- releases what the library created: on every device, waits
 * for and destroys the host-buffer pipeline's streams and events, and forgets
 * every per-device lookup (kernel attributes, the scratch array's address,
 * the stream-to-error-word map).  Must not run concurrently with another
 * call of the library.  The library stays usable: a later call re-creates
 * what it needs.  Call it before cudaDeviceReset (a reset replaces the
 * module's arrays and attributes, so cached lookups would be stale).  The
 * calling thread's current device is left as it was.
 */
void h3_shutdown(void);

/*
 * h3_build_coords -- packed segment table -> per-row (t, h, w) fp32.
 * Defining passages: [P1] section 4 (three axes, shared timeline, stereo
 * channel on another axis, row order carries no position); [P3] latent-frame,
 * text and clock-unit passages.
 *
 *   segs     host array of nseg segments (1 <= nseg <= H3_MAX_SEGMENTS)
 *   d_perm   device int32[n_rows]: packed row r holds logical element
 *            d_perm[r]; NULL = identity.  Entries outside [0, n_rows) are
 *            reported as H3_ERR_DEVICE_INPUT by h3_check_device_error and
 *            their rows get NaN coordinates.  That d_perm is a permutation
 *            is the caller's responsibility.
 *   n_rows   sum of the segments' rows (else H3_ERR_INVALID_ARG); 0 is allowed
 *   d_coords device float[n_rows][3], written
 * Errors: H3_ERR_INVALID_ARG for a bad table (unknown kind or flag, negative
 * count, non-positive grid/channels/t_den, values outside the exact range),
 * a row-count mismatch or a NULL d_coords with n_rows > 0.
 */
h3_status h3_build_coords(const h3_segment* segs, int32_t nseg, const int32_t* d_perm,
                          int64_t n_rows, float* d_coords, void* stream);

/*
 * h3_mmrope_qk -- rotate Q and K in one pass (three-axis MM-RoPE).
 * Defining passages: [P1] section 4; [P3] chain from the frame rescale to the
 * position grid to rotate(Q, K); [P5] H3-Omni-Transformer.
 *
 *   d_q, d_k          device bf16 inputs, layout above (batch folded into rows)
 *   d_q_out, d_k_out  device bf16 outputs, same layout and stride; may equal
 *                     the inputs (in place); must not partially overlap them.
 *                     d_q and d_q_out may both be NULL: then only K is rotated
 *                     (the partner of h3_packed_attention's fused Q rotation)
 *   d_coords          device float[n_rows][3] from h3_build_coords
 *   n_rows, n_heads   rows and heads; row_stride in elements
 *   cfg               host rotary configuration
 * Per element: the rotation is computed in fp32 from fp32 cos/sin of an fp64
 * angle (fp64 coordinate x fp64 inverse frequency), rounded to bf16 (RNE).
 * Errors: H3_ERR_INVALID_ARG (NULL pointer with n_rows > 0, bad cfg, bad
 * sizes); H3_ERR_UNSUPPORTED (head_dim != 128, stride not a multiple of 8,
 * pointer not 16-byte aligned).
 */
h3_status h3_mmrope_qk(const void* d_q, const void* d_k, void* d_q_out, void* d_k_out,
                       const float* d_coords, int64_t n_rows, int32_t n_heads,
                       int64_t row_stride, const h3_rope_cfg* cfg, void* stream);

/*
 * h3_rope_cos_sin -- the rotary table of every row: for pair p of row r,
 * d_cs[r][p] = (cos a, sin a), a = fp64(coordinate of p's axis) x fp64
 * inverse frequency of p, fp64 sincos, each rounded to fp32: exactly the
 * values h3_mmrope_qk rotates by.  Defining passages: as h3_mmrope_qk.  It is
 * the input of h3_packed_attention's fused Q rotation, which then rotates
 * with a table read instead of recomputing the trigonometry in every CTA.
 *
 *   d_coords   device float[n_rows][3] from h3_build_coords
 *   n_rows     rows (batch folded in)
 *   cfg        host rotary configuration (head_dim 128: 64 pairs per row)
 *   d_cs       device float[n_rows][64][2], 16-byte aligned, written
 * Errors: H3_ERR_INVALID_ARG (NULL pointer with n_rows > 0, bad cfg);
 * H3_ERR_UNSUPPORTED (head_dim != 128, misaligned d_cs).
 */
h3_status h3_rope_cos_sin(const float* d_coords, int64_t n_rows, const h3_rope_cfg* cfg, float* d_cs,
                          void* stream);

/*
 * h3_packed_attention -- full (non-causal, unmasked) softmax attention over
 * all packed rows, per batch and head:  O = softmax(Q K^T * scale) V.
 * Defining passages: [P1] sections 2 and 6 (one packed sequence, full
 * attention); [P3] bidirectional-attention passage.
 *
 *   d_q, d_k, d_v   device bf16 [batch][n_rows][n_heads][128] (Q, K already
 *                   rotated when d_coords is NULL)
 *   d_o             device bf16 output, same layout and row_stride
 *   d_lse           device float[batch][n_heads][n_rows] natural-log row
 *                   log-sum-exp of the scaled logits, or NULL
 *   d_rope_cs, cfg  NULL: Q and K arrive rotated.  Non-NULL (device float
 *                   [batch][n_rows][64][2] from h3_rope_cos_sin, 16-byte aligned;
 *                   host cfg for its pair layout): Q arrives UNROTATED and each
 *                   CTA rotates its Q tiles in shared memory as they are loaded,
 *                   with the table's (cos, sin) and exactly the arithmetic of
 *                   h3_mmrope_qk (so O is identical to rotating first); K must
 *                   already be rotated (h3_mmrope_qk with d_q = NULL).  Rotating K
 *                   here would repeat the work in every query-tile CTA of a head.
 *   softmax_scale   > 0, or <= 0 for 1/sqrt(head_dim)
 * Arithmetic: bf16 tensor-core products with fp32 accumulation (tcgen05),
 * fp32 online softmax, P rounded to bf16 for the P.V product, O rounded to
 * bf16.  All waits inside the kernel are bounded; on expiry the kernel stops
 * and h3_check_device_error returns H3_ERR_TIMEOUT.
 * Errors: H3_ERR_INVALID_ARG (NULL pointers with n_rows > 0, n_rows >= 2^31,
 * batch or n_heads < 1, bad stride, bad cfg with d_rope_cs); H3_ERR_UNSUPPORTED
 * (head_dim != 128, misaligned pointer or stride).
 */
h3_status h3_packed_attention(const void* d_q, const void* d_k, const void* d_v, void* d_o,
                              float* d_lse, const float* d_rope_cs, const h3_rope_cfg* cfg,
                              int32_t batch, int64_t n_rows, int32_t n_heads, int32_t head_dim,
                              int64_t row_stride, float softmax_scale, void* stream);

/*
 * h3_adaln_modulate -- per-row AdaLN modulation of the layer input, the step
 * before the attention projections:  y = LayerNorm(x) * (1 + scale[e]) + shift[e]
 * with e = timestep_index[row] * 3 + token_tag[row].
 * Defining passages: [P3] AdaLN passage (computed scale and shift; a table
 * indexed by (noise level, modality) with adaln_indices = timestep_indices * 3
 * + token_tags, looked up per row); [P1] section 5 (a small table of unique
 * timesteps and modalities, gathered for each row).
 *
 *   d_x, d_y           device bf16 [n_rows][hidden] with row strides x_row_stride,
 *                      y_row_stride (elements, multiples of 8; 16-byte aligned);
 *                      d_y may equal d_x (in place)
 *   d_timestep_index   device int32[n_rows]; d_token_tag device int32[n_rows]
 *                      (0 text, 1 video, 2 audio)
 *   d_table            device fp32 [n_entries][2][hidden]: [e][0] = shift,
 *                      [e][1] = scale
 *   eps                LayerNorm epsilon (biased variance; no affine of its own)
 * Arithmetic: fp32 statistics and modulation, output rounded to bf16.  A row
 * whose e falls outside [0, n_entries) gets NaN and H3_ERR_DEVICE_INPUT is
 * reported by h3_check_device_error.
 * Errors: H3_ERR_INVALID_ARG (sizes, NULL pointers, eps); H3_ERR_UNSUPPORTED
 * (hidden not a multiple of 8 or above 8192, misaligned pointer or stride).
 */
h3_status h3_adaln_modulate(const void* d_x, void* d_y, const int32_t* d_timestep_index,
                            const int32_t* d_token_tag, const float* d_table, int32_t n_entries, int64_t n_rows,
                            int32_t hidden, int64_t x_row_stride, int64_t y_row_stride, float eps, void* stream);

/*
 * Device workspace, in bytes, that h3_packed_mmrope_attention_host needs for
 * n_rows x n_heads (Q, K, V, O copies, coordinates and the permutation,
 * each 256-byte aligned).  Returns 0 for invalid sizes.
 */
uint64_t h3_host_workspace_bytes(int64_t n_rows, int32_t n_heads);

/*
 * h3_packed_mmrope_attention_host -- the whole path (coords, MM-RoPE on Q and
 * K, full attention) for one packed sequence whose Q, K, V and O live in HOST
 * memory.  Same operation and arithmetic as h3_build_coords + h3_mmrope_qk +
 * h3_packed_attention (same passages), pipelined over chunks of heads: while
 * chunk c is rotated and attended on the GPU, chunk c+1 is copied in and
 * chunk c-1's O is copied out, on two internal copy streams ordered by events.
 *
 *   segs, nseg        host segment table (as h3_build_coords)
 *   h_perm            host int32[n_rows] row permutation, or NULL
 *   h_q, h_k, h_v     host bf16 [n_rows][n_heads][128], contiguous; pinned
 *                     memory (cudaHostAlloc / cudaHostRegister) for the copies
 *                     to overlap, pageable memory works but serialises
 *   h_o               host bf16 output, same layout
 *   d_work            device workspace of h3_host_workspace_bytes() bytes,
 *                     256-byte aligned, owned by the caller; contents undefined
 *                     after the call
 *   heads_per_chunk   0 = chosen by the library (chunks whose CTA count fills
 *                     whole waves of SMs, the last few heads in halving
 *                     chunks so that little work remains after the last copy
 *                     in), else 1..n_heads heads per chunk
 *   cfg               host rotary configuration
 *   stream            work starts after everything already queued on `stream`;
 *                     the call returns once all work is queued, and `stream`
 *                     is ordered after the last copy out: synchronise `stream`
 *                     to wait for h_o.  Host buffers must stay valid until then.
 * Errors: as the three calls it composes; H3_ERR_INVALID_ARG for a NULL or
 * misaligned workspace; H3_ERR_UNSUPPORTED if the chunk plan needs more than
 * 64 chunks (always when heads_per_chunk < n_heads / 64; with 0 the library's
 * chunks hold 2 to 8 heads); H3_ERR_CUDA if an internal stream or event cannot be
 * created (they are created once per device and kept until h3_shutdown).
 * Every argument, the segment table included, is checked before anything is
 * queued.  If a CUDA call fails after copies were queued, `stream` is still
 * ordered after every queued copy before the error is returned, so
 * synchronising `stream` makes the host buffers safe to release.
 */
h3_status h3_packed_mmrope_attention_host(const h3_segment* segs, int32_t nseg, const int32_t* h_perm,
                                          const void* h_q, const void* h_k, const void* h_v, void* h_o,
                                          void* d_work, int64_t n_rows, int32_t n_heads,
                                          int32_t heads_per_chunk, const h3_rope_cfg* cfg, void* stream);

/* Size of the fixed device scratch used by h3_packed_mmrope_attention_host_noalloc. */
#define H3_NOALLOC_SCRATCH_BYTES (64ull << 20)

/*
 * h3_packed_mmrope_attention_host_noalloc -- the same computation as
 * h3_packed_mmrope_attention_host, for callers that cannot allocate device
 * memory themselves.  The pages describe no such call; it exists for
 * integration.  Typical callers that cannot allocate: code running inside a
 * host framework that owns the device's memory pool and does not allow raw
 * cudaMalloc next to it; latency-bound loops where an allocation (which can
 * synchronise the device) is not acceptable; plugins that are handed pointers
 * but no allocator.
 *
 * Instead of a caller-provided workspace it uses one fixed scratch array of
 * H3_NOALLOC_SCRATCH_BYTES (64 MiB) that lives in the library's device code:
 * every GPU that loads the library holds this memory until the process exits.
 * The call allocates nothing: no cudaMalloc, no cudaFree, no streams, no
 * events; all copies and kernels are queued in order on `stream` (no overlap
 * between copies and compute, unlike the workspace variant).
 *
 *   arguments      as h3_packed_mmrope_attention_host, without d_work and
 *                  heads_per_chunk
 *   size limit     h3_host_workspace_bytes(n_rows, n_heads) must not exceed
 *                  H3_NOALLOC_SCRATCH_BYTES, else H3_ERR_TOO_LARGE and nothing
 *                  is queued (about 65k row-heads: e.g. 4,584 rows x 8 heads)
 *   first call     the first call on each device looks up the scratch
 *                  array's device address (cudaGetSymbolAddress) and caches
 *                  it until h3_shutdown (h3_init does the same up front);
 *                  make that first call before any stream capture, and call
 *                  h3_shutdown before a cudaDeviceReset
 *   sharing        every call on a device uses the same scratch and leaves its
 *                  contents behind; nothing in it has to start at zero (each
 *                  call writes every byte it later reads).  Calls whose GPU
 *                  work overlaps in time (different streams, or different host
 *                  threads) race on the scratch: serialise them.
 */
h3_status h3_packed_mmrope_attention_host_noalloc(const h3_segment* segs, int32_t nseg, const int32_t* h_perm,
                                                  const void* h_q, const void* h_k, const void* h_v, void* h_o,
                                                  int64_t n_rows, int32_t n_heads, const h3_rope_cfg* cfg,
                                                  void* stream);

/*
 * Read and clear the error word of `stream` on the current device in one
 * atomic step ordered after the work already queued on `stream`, then
 * synchronise `stream`.  Every kernel the library launches records its faults
 * in the word of the stream it was launched on, so a check reports only that
 * stream's faults: distinct streams may be checked from distinct threads.
 * The library keeps 255 such words per device, handed out to streams in the
 * order it first sees them; streams beyond the 255th share one further word.
 * Returns H3_OK, H3_ERR_TIMEOUT, H3_ERR_DEVICE_INPUT or H3_ERR_CUDA.
 */
h3_status h3_check_device_error(void* stream);

/*
 * Limit, in nanoseconds of device global time, of every bounded wait inside
 * the attention kernel (process-wide; default 2e9 = 2 s).  0 restores the
 * default.  Used by tests to force the timeout path.
 */
h3_status h3_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* H3_H_ */
