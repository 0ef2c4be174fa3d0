"""Helpers shared by the GPU parity tests (comparison rules and set-up)."""
import numpy as np
import torch

# Tolerances of the parity contract for floating point: bf16 weights, fp32
# accumulation against the fp64 oracle.  Both must hold.
MAX_ABS = 3e-2
REL_L2 = 1e-2
# An emitted id may differ from the oracle's only where the oracle's top-2
# logit margin is below this.
NEAR_TIE = 1e-2


def close_report(got, ref):
    got = np.asarray(got, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), "non-finite value on the CUDA path"
    diff = got - ref
    maxabs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return maxabs, rel


def assert_close(got, ref, what=""):
    maxabs, rel = close_report(got, ref)
    assert maxabs <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {maxabs:.3g} rel-L2 {rel:.3g}"
    return maxabs, rel


def assert_id(gpu_id: int, oracle_result, what=""):
    if gpu_id != oracle_result.token:
        assert oracle_result.margin < NEAR_TIE, (
            f"{what}: id {gpu_id} != oracle {oracle_result.token} (margin {oracle_result.margin:.3g})")


def i32(vals, device="cuda"):
    return torch.tensor(list(vals), dtype=torch.int32, device=device)


def bf16_values(t):
    """bf16 device/host tensor -> float64 numpy."""
    return t.detach().to("cpu").double().numpy()
