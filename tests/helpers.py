"""Shared test helpers: device transfer, oracle comparison, the accuracy gates.

Gates (relative Frobenius error <= 1e-3 and max |err| <= 1e-2 * max|ref|) apply to
f32-output runs against the f64 oracle and to bf16-output runs against the oracle's
result rounded to bf16 (nearest even); a bf16 output cannot be closer to the f64 value
than its own rounding, which alone is ~1.6e-3 relative.
"""
from __future__ import annotations

import numpy as np
import torch

REL_FRO = 1e-3
MAX_REL = 1e-2


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def dev(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """numpy -> CUDA tensor of `dtype`, reinterpreting bit patterns for 16-bit types."""
    a = np.ascontiguousarray(a)
    if dtype in (torch.bfloat16, torch.float16):
        t = torch.from_numpy(a.view(np.int16)).view(dtype)
    else:
        t = torch.from_numpy(a).to(dtype)
    return t.cuda()


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def out_to_f64(y: torch.Tensor) -> np.ndarray:
    if y.dtype == torch.bfloat16:
        return bf16_to_f32(bits16(y)).astype(np.float64)
    return y.detach().cpu().numpy().astype(np.float64)


def gate(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Assert the two accuracy gates; return (rel_fro, max_rel) for reporting."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs (kernel did not write?)"
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    mref = np.max(np.abs(ref)) if ref.size else 0.0
    mx = np.max(np.abs(err)) / mref if mref > 0 else np.max(np.abs(err), initial=0.0)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_REL, f"{what}: max error {mx:.3e} of max|ref| > {MAX_REL}"
    return rel, mx


def gate_output(y: torch.Tensor, ref64: np.ndarray, oracle, what: str = ""):
    """Gate a kernel output against the f64 oracle under the rule for its dtype."""
    got = out_to_f64(y)
    if y.dtype == torch.bfloat16:
        ref = bf16_to_f32(oracle.f64_to_bf16(ref64)).astype(np.float64)
    else:
        ref = ref64
    return gate(got, ref, what)


def nan_filled(shape, dtype, pad: int = 64):
    """An output tensor pre-filled with NaN, followed by `pad` canary elements.

    Returns (y_view, full_buffer); the canary is the buffer's tail."""
    M, N = shape
    buf = torch.full((M * N + pad,), float("nan"), dtype=dtype, device="cuda")
    buf[M * N:] = 12288.0
    return buf[: M * N].view(M, N), buf


def canary_intact(buf: torch.Tensor, n: int) -> bool:
    tail = buf[n:].float().cpu().numpy()
    return bool(np.all(tail == np.float32(12288.0)))


def worst_blocks(got: np.ndarray, ref: np.ndarray, tok: int = 256, rows: int = 32, top: int = 3):
    """The `top` output blocks (token tile of `tok` x weight rows of `rows`) with the largest
    relative Frobenius error, as (token tile, row block, rel error) -- a striped failure
    (one TMEM lane quarter of a tile, one CTA's rows) then shows up by name."""
    M, N = ref.shape
    out = []
    for m0 in range(0, M, tok):
        for n0 in range(0, N, rows):
            r = ref[m0:m0 + tok, n0:n0 + rows]
            e = got[m0:m0 + tok, n0:n0 + rows] - r
            nr = np.linalg.norm(r)
            out.append((m0 // tok, n0 // rows, float(np.linalg.norm(e) / nr if nr > 0 else np.linalg.norm(e))))
    out.sort(key=lambda t: -t[2])
    return out[:top]


def gate_full(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """gate() over a whole output matrix [M, N]; on failure the message names the worst
    (256-token tile, 32-row block) pieces."""
    try:
        return gate(got, ref, what)
    except AssertionError as e:
        blocks = worst_blocks(np.asarray(got, np.float64), np.asarray(ref, np.float64))
        raise AssertionError(f"{e}; worst (token tile, 32-row block, rel err): {blocks}") from None
