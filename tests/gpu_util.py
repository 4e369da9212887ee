"""Helpers shared by the GPU parity tests: moving seeded numpy inputs onto the
device and comparing outputs with the tolerances the tests state."""

from __future__ import annotations

import numpy as np
import torch

# Attention tolerances for bf16 inputs with binary32 accumulation: relative
# Frobenius error of O, max abs error of O, max abs error of the natural-log
# LSE.
ATTN_REL_FRO = 1e-2
ATTN_MAX_ABS = 3e-2
LSE_MAX_ABS = 1e-3


def to_dev(a: np.ndarray, dtype: str = "auto") -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint8)


def f32_bits(t) -> np.ndarray:
    a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else t
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_attention_close(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray,
                           what: str = ""):
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), f"{what}: -inf pattern of lse differs"
    if o_ref.size:
        den = np.linalg.norm(o_ref)
        rel = np.linalg.norm(o_gpu - o_ref) / den if den > 0 else np.linalg.norm(o_gpu)
        mx = np.max(np.abs(o_gpu - o_ref))
        assert rel <= ATTN_REL_FRO, f"{what}: rel Frobenius {rel:.3e}"
        assert mx <= ATTN_MAX_ABS, f"{what}: max abs {mx:.3e}"
    if fin.any():
        lmx = np.max(np.abs(np.asarray(lse_gpu, np.float64)[fin] - lse_ref[fin]))
        assert lmx <= LSE_MAX_ABS, f"{what}: lse max abs {lmx:.3e}"
