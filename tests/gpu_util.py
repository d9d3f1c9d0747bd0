"""Helpers shared by the GPU parity tests: seeded inputs, bf16 round trips, comparison metrics."""
import numpy as np
import torch

from gpt_decoder_pretraining_b200.inputs import round_to_bf16


def bf16_tensor(a: np.ndarray, device="cuda"):
    """Exact upload of bf16-representable float32 values."""
    return torch.from_numpy(np.ascontiguousarray(round_to_bf16(a))).to(device).to(torch.bfloat16)


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def randn(rng, *shape, scale=1.0):
    return round_to_bf16(rng.standard_normal(shape).astype(np.float32) * np.float32(scale)).astype(np.float64)


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb + 1e-300))


def assert_close_rel(got, ref, rel=1e-2, cos=0.9999, what="", atol=1e-6):
    """max |got − ref| ≤ rel · max |ref| + atol  and  cosine(got, ref) ≥ cos.

    When the reference is (numerically) zero everywhere — e.g. dq of a single-key softmax — only
    the absolute bound applies, since the cosine of rounding noise is meaningless.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= rel * scale + atol, f"{what}: max err {err:.3e} vs scale {scale:.3e} (rel {rel})"
    if scale > 100 * atol:
        c = cosine(got, ref)
        assert c >= cos, f"{what}: cosine {c:.6f} < {cos}"


def f32_accum_rel(K: int) -> float:
    """Relative tolerance (of max |C|) for an fp32-accumulated product over K exactly representable
    bf16 terms.  Each partial sum is rounded to 2^-24 of its size; with terms of random sign the
    rounding errors add like a random walk, so the error of C grows like √K · 2^-24 times the
    typical partial sum, which is about max |C| / 3 for these inputs.  5e-7·√K is about 25× that
    estimate; the products of a tile's K loop accumulate in the tensor core in its own order."""
    return max(1e-5, 5e-7 * float(np.sqrt(K)))
