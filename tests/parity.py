"""Helpers for GPU-vs-oracle parity tests (CPU side only; no method arithmetic here)."""
import numpy as np
import torch

import oracle
from workloads import bf16_bits

# Tolerance for bf16 inputs with fp32 accumulation (max / mean absolute error).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def host_arrays(inp):
    """The oracle's view of a workload: raw bf16 bits and int arrays on the host."""
    return dict(q=bf16_bits(inp.q), k=bf16_bits(inp.k_pages), v=bf16_bits(inp.v_pages),
                bt=inp.block_table.cpu().numpy(), sl=inp.seq_lens.cpu().numpy(),
                scale=inp.scale)


def oracle_out(h):
    return oracle.paged_decode_attention(h["q"], h["k"], h["v"], h["bt"], h["sl"], h["scale"])


def oracle_rows(h, rows):
    return oracle.paged_decode_attention_rows(h["q"], h["k"], h["v"], h["bt"], h["sl"], h["scale"], rows)


def gpu_f64(out: torch.Tensor) -> np.ndarray:
    return out.detach().float().cpu().double().numpy()


def assert_close(got: np.ndarray, want: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    err = np.abs(got - want)
    worst = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} at {worst}"
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())
