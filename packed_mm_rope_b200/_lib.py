"""ctypes binding of libh3 (argument marshalling only).

Every function here forwards to the C ABI in include/h3.h with the same name;
the computation runs in the library's CUDA kernels.  There is no fallback: if
libh3.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libh3.so")

(H3_OK, H3_ERR_INVALID_ARG, H3_ERR_UNSUPPORTED, H3_ERR_CUDA, H3_ERR_TIMEOUT, H3_ERR_DEVICE_INPUT,
 H3_ERR_TOO_LARGE) = range(7)
H3_NOALLOC_SCRATCH_BYTES = 64 << 20
H3_SEG_TEXT, H3_SEG_VIDEO, H3_SEG_AUDIO = 0, 1, 2
H3_FLAG_TEXT_T_ONLY, H3_FLAG_AUDIO_CHANNEL_H, H3_FLAG_VIDEO_CANVAS = 1, 2, 4
H3_MAX_SEGMENTS = 64

EXPORTED = ("h3_status_str", "h3_version", "h3_build_coords", "h3_mmrope_qk", "h3_rope_cos_sin",
            "h3_packed_attention", "h3_check_device_error", "h3_set_wait_limit_ns",
            "h3_host_workspace_bytes", "h3_packed_mmrope_attention_host",
            "h3_packed_mmrope_attention_host_noalloc", "h3_adaln_modulate", "h3_init", "h3_shutdown")


class h3_segment(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("kind", "count", "grid_h", "grid_w", "channels", "t_off_num", "t_step_num", "t_den", "flags")]


class h3_rope_cfg(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_double), ("head_dim", ctypes.c_int32), ("sec_t", ctypes.c_int32),
                ("sec_h", ctypes.c_int32), ("sec_w", ctypes.c_int32), ("pair_layout", ctypes.c_int32),
                ("freq_rule", ctypes.c_int32)]


class H3Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libh3.so (built in-tree by packed_mm_rope_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libh3.so not built: {path} (run python -m packed_mm_rope_b200.build)")
    lib = ctypes.CDLL(path)
    P, I32, I64, F32, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64
    lib.h3_status_str.restype = ctypes.c_char_p
    lib.h3_status_str.argtypes = [I32]
    lib.h3_version.restype = I32
    lib.h3_version.argtypes = []
    lib.h3_build_coords.restype = I32
    lib.h3_build_coords.argtypes = [ctypes.POINTER(h3_segment), I32, P, I64, P, P]
    lib.h3_mmrope_qk.restype = I32
    lib.h3_mmrope_qk.argtypes = [P, P, P, P, P, I64, I32, I64, ctypes.POINTER(h3_rope_cfg), P]
    lib.h3_rope_cos_sin.restype = I32
    lib.h3_rope_cos_sin.argtypes = [P, I64, ctypes.POINTER(h3_rope_cfg), P, P]
    lib.h3_packed_attention.restype = I32
    lib.h3_packed_attention.argtypes = [P, P, P, P, P, P, ctypes.POINTER(h3_rope_cfg), I32, I64, I32, I32,
                                        I64, F32, P]
    lib.h3_check_device_error.restype = I32
    lib.h3_check_device_error.argtypes = [P]
    lib.h3_set_wait_limit_ns.restype = I32
    lib.h3_set_wait_limit_ns.argtypes = [U64]
    lib.h3_host_workspace_bytes.restype = U64
    lib.h3_host_workspace_bytes.argtypes = [I64, I32]
    lib.h3_packed_mmrope_attention_host.restype = I32
    lib.h3_packed_mmrope_attention_host.argtypes = [ctypes.POINTER(h3_segment), I32, P, P, P, P, P, P, I64, I32,
                                                    I32, ctypes.POINTER(h3_rope_cfg), P]
    lib.h3_packed_mmrope_attention_host_noalloc.restype = I32
    lib.h3_packed_mmrope_attention_host_noalloc.argtypes = [ctypes.POINTER(h3_segment), I32, P, P, P, P, P, I64,
                                                            I32, ctypes.POINTER(h3_rope_cfg), P]
    lib.h3_init.restype = I32
    lib.h3_init.argtypes = [I32]
    lib.h3_shutdown.restype = None
    lib.h3_shutdown.argtypes = []
    lib.h3_adaln_modulate.restype = I32
    lib.h3_adaln_modulate.argtypes = [P, P, P, P, P, I32, I64, I32, I64, I64, F32, P]
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load().h3_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != H3_OK:
        raise H3Error(status, where)


def segment_array(segments):
    """Python segments (objects with the h3_segment field names, or 9-tuples) -> ctypes array."""
    arr = (h3_segment * max(len(segments), 1))()
    for i, s in enumerate(segments):
        vals = s.as_tuple() if hasattr(s, "as_tuple") else tuple(s)
        for (name, _), v in zip(h3_segment._fields_, vals):
            setattr(arr[i], name, int(v))
    return arr


def rope_cfg(theta=10000.0, head_dim=128, sections=(32, 48, 48), pair_layout=0, freq_rule=0) -> h3_rope_cfg:
    return h3_rope_cfg(float(theta), int(head_dim), int(sections[0]), int(sections[1]), int(sections[2]),
                       int(pair_layout), int(freq_rule))


def h3_build_coords(segments, d_perm: int, n_rows: int, d_coords: int, stream: int = 0) -> None:
    arr = segment_array(segments)
    _check(load().h3_build_coords(arr, len(segments), d_perm or None, n_rows, d_coords or None,
                                  stream or None), "h3_build_coords")


def h3_mmrope_qk(d_q: int, d_k: int, d_q_out: int, d_k_out: int, d_coords: int, n_rows: int, n_heads: int,
                 row_stride: int, cfg: h3_rope_cfg, stream: int = 0) -> None:
    _check(load().h3_mmrope_qk(d_q or None, d_k or None, d_q_out or None, d_k_out or None, d_coords or None,
                               n_rows, n_heads, row_stride, ctypes.byref(cfg), stream or None), "h3_mmrope_qk")


def h3_rope_cos_sin(d_coords: int, n_rows: int, cfg: h3_rope_cfg, d_cs: int, stream: int = 0) -> None:
    _check(load().h3_rope_cos_sin(d_coords or None, n_rows, ctypes.byref(cfg), d_cs or None, stream or None),
           "h3_rope_cos_sin")


def h3_packed_attention(d_q: int, d_k: int, d_v: int, d_o: int, d_lse: int, batch: int, n_rows: int,
                        n_heads: int, row_stride: int, softmax_scale: float = 0.0, head_dim: int = 128,
                        d_rope_cs: int = 0, cfg: h3_rope_cfg | None = None, stream: int = 0) -> None:
    _check(load().h3_packed_attention(d_q or None, d_k or None, d_v or None, d_o or None, d_lse or None,
                                      d_rope_cs or None, ctypes.byref(cfg) if cfg is not None else None,
                                      batch, n_rows, n_heads, head_dim, row_stride, softmax_scale,
                                      stream or None), "h3_packed_attention")


def h3_host_workspace_bytes(n_rows: int, n_heads: int) -> int:
    return int(load().h3_host_workspace_bytes(n_rows, n_heads))


def h3_packed_mmrope_attention_host(segments, h_perm: int, h_q: int, h_k: int, h_v: int, h_o: int, d_work: int,
                                    n_rows: int, n_heads: int, cfg: h3_rope_cfg, heads_per_chunk: int = 0,
                                    stream: int = 0) -> None:
    arr = segment_array(segments)
    _check(load().h3_packed_mmrope_attention_host(arr, len(segments), h_perm or None, h_q or None, h_k or None,
                                                  h_v or None, h_o or None, d_work or None, n_rows, n_heads,
                                                  heads_per_chunk, ctypes.byref(cfg), stream or None),
           "h3_packed_mmrope_attention_host")


def h3_packed_mmrope_attention_host_noalloc(segments, h_perm: int, h_q: int, h_k: int, h_v: int, h_o: int,
                                            n_rows: int, n_heads: int, cfg: h3_rope_cfg, stream: int = 0) -> None:
    """The host-buffer call without a caller workspace (see include/h3.h)."""
    arr = segment_array(segments)
    _check(load().h3_packed_mmrope_attention_host_noalloc(arr, len(segments), h_perm or None, h_q or None,
                                                          h_k or None, h_v or None, h_o or None, n_rows, n_heads,
                                                          ctypes.byref(cfg), stream or None),
           "h3_packed_mmrope_attention_host_noalloc")


def h3_adaln_modulate(d_x: int, d_y: int, d_ts: int, d_tags: int, d_table: int, n_entries: int, n_rows: int,
                      hidden: int, x_row_stride: int, y_row_stride: int, eps: float = 1e-6, stream: int = 0) -> None:
    _check(load().h3_adaln_modulate(d_x or None, d_y or None, d_ts or None, d_tags or None, d_table or None,
                                    n_entries, n_rows, hidden, x_row_stride, y_row_stride, eps, stream or None),
           "h3_adaln_modulate")


def h3_check_device_error(stream: int = 0) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(load().h3_check_device_error(stream or None))


def h3_init(device: int = 0) -> None:
    """Up-front set-up of one device (optional; every call also does it lazily)."""
    _check(load().h3_init(int(device)), "h3_init")


def h3_shutdown() -> None:
    """Release the library's streams and events on every device."""
    load().h3_shutdown()


def h3_set_wait_limit_ns(ns: int) -> None:
    _check(load().h3_set_wait_limit_ns(int(ns)), "h3_set_wait_limit_ns")
