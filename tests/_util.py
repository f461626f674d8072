"""Shared helpers of the GPU parity tests (comparison metrics, input transfer)."""

import numpy as np

import synth

# Acceptance bars against the fp64 oracle (fp32 accumulation on the GPU, bf16 outputs)
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to_f64(t) -> np.ndarray:
    """A CUDA/CPU torch tensor (bf16 or fp32) -> fp64 numpy."""
    import torch

    return t.detach().to(torch.float64).cpu().numpy()


def bits(t) -> np.ndarray:
    """bf16 torch tensor -> uint16 bit patterns (numpy)."""
    import torch

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def dev_bf16(bits_np, device="cuda"):
    return synth.to_torch_bf16(bits_np).to(device)


def rel_l2(a, b) -> float:
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


def assert_out_close(got, ref, what="O"):
    err = np.max(np.abs(got - ref)) if got.size else 0.0
    rl = rel_l2(got, ref)
    assert err <= O_MAX_ABS and rl <= O_REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rl:.3e}"


def assert_lse_close(got, ref):
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "LSE finiteness differs"
    assert np.all(got[~fin] == ref[~fin]), "LSE -inf rows differ"
    if fin.any():
        err = np.max(np.abs(got[fin] - ref[fin]))
        assert err <= LSE_MAX_ABS, f"LSE max-abs {err:.3e}"
