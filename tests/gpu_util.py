"""Helpers for the GPU parity tests (device copies and tolerance checks)."""
import numpy as np

ATTN_MAX_ABS = 2e-2    # stated tolerance: max |err| of O against the fp64 oracle
ATTN_MEAN_ABS = 2e-3   # stated tolerance: mean |err|
ATTN_REL = 1e-2        # extra: ||O - O_ref|| / ||O_ref|| (bf16 rounding of rotated Q/K, P and O ~ 3e-3)


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def check_rope(got_bits: np.ndarray, exact: np.ndarray, x_in: np.ndarray, pair_layout: int = 0,
               dang: np.ndarray | None = None):
    """|gpu - exact| <= 1 bf16 ulp(exact) + (2^-21 + dang) (|x0| + |x1|) per element.

    2^-21 bounds the fp32 evaluation x0*c - x1*s with c, s rounded to fp32 (a
    few units of 2^-24 relative to the pair's magnitude).  ``dang`` [rows, D/2]
    is |angle(fp32 coordinate) - angle(exact coordinate)|: the library rotates
    by its fp32 coordinates, the oracle by the exact rationals, and a rotation
    error of dang moves each output by at most dang (|x0| + |x1|).  The ulp
    term is the final rounding to bf16 plus one possible flip at a rounding
    boundary.  Returns (fraction of elements equal to RNE(exact), max error in
    ulps).
    """
    got = bf16_bits_to_f64(got_bits)
    if pair_layout == 0:
        mag = np.abs(x_in[..., 0::2]) + np.abs(x_in[..., 1::2])
        mag = np.repeat(mag, 2, axis=-1)
    else:
        h = x_in.shape[-1] // 2
        mag = np.abs(x_in[..., :h]) + np.abs(x_in[..., h:])
        mag = np.concatenate([mag, mag], axis=-1)
    err = np.abs(got - exact)
    slack = 2.0 ** -21
    if dang is not None:
        d = dang.reshape(dang.shape[:1] + (1,) * (x_in.ndim - 2) + dang.shape[1:])
        d = np.repeat(d, 2, axis=-1) if pair_layout == 0 else np.concatenate([d, d], axis=-1)
        slack = slack + d
    bound = bf16_ulp(exact) + slack * mag
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} rotated elements outside 1 ulp (worst {err[bad].max():.3e})"
    import workload as W
    rne = bf16_bits_to_f64(W.bf16_bits_rne(exact))
    return float((got == rne).mean()), float((err / bf16_ulp(exact)).max())


def check_attention(got: np.ndarray, ref: np.ndarray, label: str = "", logit_scale: float = 1.0):
    """Stated tolerances; ``logit_scale`` widens the absolute ones for inputs whose
    logits are that many times larger than N(0,1) Q/K give: the library rounds the
    rotated Q and K to bf16, so each logit carries an error proportional to its
    own magnitude, and O moves by that error times |O| (which is O(1) once the
    softmax concentrates on a few keys)."""
    err = np.abs(got - ref)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    msg = f"{label} max|err| {err.max():.3e} mean|err| {err.mean():.3e} rel {rel:.3e}"
    assert np.isfinite(got).all(), label + " non-finite output"
    assert err.max() <= ATTN_MAX_ABS * logit_scale, msg
    assert err.mean() <= ATTN_MEAN_ABS * logit_scale, msg
    assert rel <= ATTN_REL, msg
    return float(err.max()), float(err.mean()), rel
