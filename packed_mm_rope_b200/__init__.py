"""packed_mm_rope_b200 -- packed multimodal MM-RoPE attention for B200 (sm_100a).

Thin Python layer over the C ABI of ``libh3.so`` (include/h3.h).  PyTorch is
used only to hold device memory and to name the current CUDA stream; every
step of the path runs in the library's CUDA kernels:

* ``h3_build_coords``     packed segment table -> per-row (t, h, w) fp32
* ``h3_mmrope_qk``        three-axis rotary rotation of bf16 Q and K
* ``h3_rope_cos_sin``     the per-row rotary (cos, sin) table of the fused Q rotation
* ``h3_packed_attention`` full softmax attention over the packed rows

The library is loaded on first use (``load()``, or any call below) and a
missing or stale ``libh3.so`` raises there; there is no CPU or eager-PyTorch
fallback.  Importing the package itself does not load it, so that
``python -m packed_mm_rope_b200.build`` can (re)build a missing library.
"""
from __future__ import annotations

from . import _lib
from ._lib import (H3Error, H3_OK, H3_ERR_INVALID_ARG, H3_ERR_UNSUPPORTED, H3_ERR_CUDA,  # noqa: F401
                   H3_ERR_TIMEOUT, H3_ERR_DEVICE_INPUT, H3_ERR_TOO_LARGE, h3_adaln_modulate,
                   h3_build_coords, h3_check_device_error, h3_init, h3_shutdown,
                   h3_host_workspace_bytes, h3_mmrope_qk, h3_packed_attention, h3_packed_mmrope_attention_host,
                   h3_rope_cos_sin,
                   h3_set_wait_limit_ns, rope_cfg, status_str)

load = _lib.load


def _stream(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _on_device(t, what: str) -> None:
    """Raise unless ``t`` lives on the current CUDA device (the library dereferences it there)."""
    import torch
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"{what} must be on the current CUDA device")


def _exact(t, dtype, shape, what: str) -> None:
    """Raise unless ``t`` is a contiguous tensor of exactly this dtype and shape."""
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{what} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _row_layout(x):
    """(batch, n_rows, n_heads, row_stride) of a [.., N, H, 128] bf16 view."""
    import torch
    if x.dtype != torch.bfloat16 or not x.is_cuda:
        raise TypeError("expected a CUDA bf16 tensor")
    _on_device(x, "Q, K, V and O")
    if x.dim() not in (3, 4) or x.shape[-1] != 128 or x.stride(-1) != 1 or x.stride(-2) != 128:
        raise ValueError("expected [N, H, 128] or [B, N, H, 128] with heads contiguous")
    n, h = x.shape[-3], x.shape[-2]
    rs = x.stride(-3)
    b = x.shape[0] if x.dim() == 4 else 1
    if x.dim() == 4 and b > 1 and x.stride(0) != n * rs:
        raise ValueError("batch stride must be n_rows * row_stride")
    return b, n, h, rs


def build_coords(segments, n_rows: int, perm=None, out=None, stream=None):
    """fp32 [n_rows, 3] coordinates on the current device."""
    import torch
    if out is None:
        out = torch.empty((n_rows, 3), dtype=torch.float32, device="cuda")
    _exact(out, torch.float32, (n_rows, 3), "out")
    _on_device(out, "out")
    p = 0
    if perm is not None:
        if perm.dtype != torch.int32 or not perm.is_cuda or perm.numel() != n_rows or not perm.is_contiguous():
            raise ValueError("perm must be a contiguous CUDA int32 tensor of n_rows entries")
        _on_device(perm, "perm")
        p = perm.data_ptr()
    h3_build_coords(segments, p, n_rows, out.data_ptr(), _stream(stream))
    return out


def mmrope_qk(q, k, coords, q_out=None, k_out=None, theta=10000.0, sections=(32, 48, 48), pair_layout=0,
              stream=None, freq_rule=0):
    """Rotate Q and K; returns (q_out, k_out).  Pass q_out=q, k_out=k for in place.

    q=None rotates K only (returns (None, k_out)).
    """
    import torch
    b, n, h, rs = _row_layout(k)
    if q is not None and _row_layout(q) != (b, n, h, rs):
        raise ValueError("q and k layouts differ")
    if q is not None:
        q_out = torch.empty_like(q) if q_out is None else q_out
        if _row_layout(q_out) != (b, n, h, rs):
            raise ValueError("outputs must share the inputs' layout")
    k_out = torch.empty_like(k) if k_out is None else k_out
    if _row_layout(k_out) != (b, n, h, rs):
        raise ValueError("outputs must share the inputs' layout")
    if coords.dtype != torch.float32 or coords.numel() != 3 * b * n or not coords.is_contiguous():
        raise ValueError("coords must be contiguous fp32 [rows, 3]")
    _on_device(coords, "coords")
    h3_mmrope_qk(q.data_ptr() if q is not None else 0, k.data_ptr(),
                 q_out.data_ptr() if q is not None else 0, k_out.data_ptr(), coords.data_ptr(), b * n, h,
                 rs, rope_cfg(theta, 128, sections, pair_layout, freq_rule), _stream(stream))
    return (q_out if q is not None else None), k_out


def rope_cos_sin(coords, out=None, theta=10000.0, sections=(32, 48, 48), pair_layout=0, freq_rule=0,
                 stream=None):
    """fp32 [rows, 64, 2] rotary (cos, sin) table of fp32 [rows, 3] coordinates."""
    import torch
    if coords.dtype != torch.float32 or coords.dim() != 2 or coords.shape[1] != 3 or not coords.is_contiguous():
        raise ValueError("coords must be contiguous fp32 [rows, 3]")
    _on_device(coords, "coords")
    n = coords.shape[0]
    if out is None:
        out = torch.empty((n, 64, 2), dtype=torch.float32, device=coords.device)
    if out.dtype != torch.float32 or out.numel() != n * 128 or not out.is_contiguous():
        raise ValueError("out must be contiguous fp32 [rows, 64, 2]")
    _on_device(out, "out")
    h3_rope_cos_sin(coords.data_ptr(), n, rope_cfg(theta, 128, sections, pair_layout, freq_rule), out.data_ptr(),
                    _stream(stream))
    return out


def packed_attention(q, k, v, out=None, lse=None, softmax_scale: float = 0.0, stream=None, rope_cs=None,
                     theta=10000.0, sections=(32, 48, 48), pair_layout=0, freq_rule=0):
    """O = softmax(Q K^T * scale) V over all packed rows, per head.

    With ``rope_cs`` (fp32 [rows, 64, 2] from ``rope_cos_sin``) Q is passed
    UNROTATED and rotated inside the kernel as its tiles are loaded; K must
    already be rotated.
    """
    import torch
    lay = _row_layout(q)
    if _row_layout(k) != lay or _row_layout(v) != lay:
        raise ValueError("q, k, v layouts differ")
    out = torch.empty_like(q) if out is None else out
    if _row_layout(out) != lay:
        raise ValueError("output must share the inputs' layout")
    b, n, h, rs = lay
    lp = 0
    if lse is not None:
        if lse.dtype != torch.float32 or lse.numel() != b * h * n or not lse.is_contiguous():
            raise ValueError("lse must be contiguous fp32 [B, H, N]")
        _on_device(lse, "lse")
        lp = lse.data_ptr()
    cp, cfg = 0, None
    if rope_cs is not None:
        if rope_cs.dtype != torch.float32 or rope_cs.numel() != 128 * b * n or not rope_cs.is_contiguous():
            raise ValueError("rope_cs must be contiguous fp32 [rows, 64, 2]")
        _on_device(rope_cs, "rope_cs")
        cp, cfg = rope_cs.data_ptr(), rope_cfg(theta, 128, sections, pair_layout, freq_rule)
    h3_packed_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lp, b, n, h, rs,
                        softmax_scale, d_rope_cs=cp, cfg=cfg, stream=_stream(stream))
    return out


def packed_mmrope_attention(segments, q, k, v, perm=None, theta=10000.0, sections=(32, 48, 48),
                            pair_layout=0, out=None, lse=None, softmax_scale: float = 0.0, stream=None,
                            fused_q_rope: bool = False, freq_rule=0):
    """The whole path on one packed sequence: coords -> rotate Q, K -> attention.

    q, k, v: [N, H, 128] bf16 on the GPU (unrotated).  Returns O [N, H, 128].
    fused_q_rope: rotate only K beforehand and Q inside the attention kernel
    (from the rows' rotary table).
    """
    n = q.shape[-3]
    coords = build_coords(segments, n, perm, stream=stream)
    if fused_q_rope:
        cs = rope_cos_sin(coords, theta=theta, sections=sections, pair_layout=pair_layout, freq_rule=freq_rule,
                          stream=stream)
        _, kr = mmrope_qk(None, k, coords, theta=theta, sections=sections, pair_layout=pair_layout,
                          stream=stream, freq_rule=freq_rule)
        return packed_attention(q, kr, v, out=out, lse=lse, softmax_scale=softmax_scale, stream=stream,
                                rope_cs=cs, theta=theta, sections=sections, pair_layout=pair_layout,
                                freq_rule=freq_rule)
    qr, kr = mmrope_qk(q, k, coords, theta=theta, sections=sections, pair_layout=pair_layout, stream=stream,
                       freq_rule=freq_rule)
    return packed_attention(qr, kr, v, out=out, lse=lse, softmax_scale=softmax_scale, stream=stream)


def host_workspace(n_rows: int, n_heads: int, device=None):
    """A device workspace (uint8 tensor) for packed_mmrope_attention_host."""
    import torch
    nbytes = h3_host_workspace_bytes(n_rows, n_heads)
    if nbytes == 0:
        raise ValueError("invalid sizes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def packed_mmrope_attention_host(segments, q, k, v, out=None, perm=None, workspace=None, theta=10000.0,
                                 sections=(32, 48, 48), pair_layout=0, heads_per_chunk: int = 0, stream=None,
                                 freq_rule=0):
    """The whole path from and to HOST memory, copies overlapped with compute.

    q, k, v: CPU bf16 [N, H, 128] contiguous tensors (pin them for overlap);
    perm: CPU int32 [N] or None.  Returns the CPU output (``out`` if given).
    Work is queued on ``stream``; synchronise it before reading the output.
    """
    import torch
    if q.dim() != 3 or q.shape[-1] != 128:
        raise ValueError("expected [N, H, 128]")
    for t in (q, k, v):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v must be contiguous CPU bf16 tensors of one shape")
    n, h = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty_like(q, pin_memory=q.is_pinned())
    if out.is_cuda:
        raise ValueError("out must be a CPU tensor")
    _exact(out, torch.bfloat16, q.shape, "out")
    if perm is not None and (perm.dtype != torch.int32 or perm.is_cuda or perm.numel() != n
                             or not perm.is_contiguous()):
        raise ValueError("perm must be a contiguous CPU int32 tensor of N entries")
    if workspace is None:
        workspace = host_workspace(n, h)
    need = h3_host_workspace_bytes(n, h)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.numel() < need:
        raise ValueError(f"workspace must be a contiguous uint8 tensor of at least {need} bytes")
    _on_device(workspace, "workspace")
    h3_packed_mmrope_attention_host(segments, perm.data_ptr() if perm is not None else 0, q.data_ptr(),
                                    k.data_ptr(), v.data_ptr(), out.data_ptr(), workspace.data_ptr(), n, h,
                                    rope_cfg(theta, 128, sections, pair_layout, freq_rule), heads_per_chunk,
                                    _stream(stream))
    return out


def adaln_modulate(x, timestep_index, token_tag, table, out=None, eps: float = 1e-6, stream=None):
    """y = LayerNorm(x) * (1 + scale[e]) + shift[e], e = timestep_index * 3 + token_tag.

    x: CUDA bf16 [N, C] (row stride a multiple of 8); timestep_index, token_tag:
    CUDA int32 [N]; table: CUDA fp32 [E, 2, C] (shift, scale).  Pass out=x for in place.
    """
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1 or not x.is_cuda:
        raise ValueError("x must be a CUDA bf16 [N, C] tensor with unit inner stride")
    n, c = x.shape
    out = torch.empty_like(x) if out is None else out
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (n, c) or out.stride(1) != 1:
        raise ValueError("out must be a bf16 [N, C] tensor with unit inner stride")
    for t, what in ((x, "x"), (out, "out")):
        _on_device(t, what)
    for t in (timestep_index, token_tag):
        if t.dtype != torch.int32 or t.numel() != n or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("indices must be contiguous CUDA int32 [N]")
        _on_device(t, "indices")
    if table.dtype != torch.float32 or table.dim() != 3 or tuple(table.shape[1:]) != (2, c) \
            or not table.is_contiguous():
        raise ValueError("table must be contiguous fp32 [E, 2, C]")
    _on_device(table, "table")
    h3_adaln_modulate(x.data_ptr(), out.data_ptr(), timestep_index.data_ptr(), token_tag.data_ptr(),
                      table.data_ptr(), table.shape[0], n, c, x.stride(0), out.stride(0), eps, _stream(stream))
    return out
