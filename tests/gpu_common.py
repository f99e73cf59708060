"""Shared helpers for the GPU parity tests (comparison against the fp64 oracle)."""
import numpy as np
import torch

from exact_attention_108_b200 import binding
from exact_attention_108_b200.workloads import make_inputs, to_f64

# Tolerances the workload definition states (forward O and LSE absolute; gradients
# relative to the largest reference magnitude of the same tensor).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3
GRAD_REL = 2e-2


def check_o(o_gpu, o_ref, what=""):
    """O max-abs <= 1e-2 and mean-abs <= 1e-3.  The max-abs bound is on the
    computation: O is delivered as bf16, and the rounding of the result itself
    to that format (half an ulp, <= 2^-8 |O|; 0.0156 at |O| = 4) comes on top."""
    err = np.abs(to_f64(o_gpu) - o_ref) if isinstance(o_gpu, torch.Tensor) else np.abs(o_gpu - o_ref)
    assert np.isfinite(err).all(), f"{what} O has non-finite values"
    excess = err - (O_MAX_ABS + 2.0 ** -8 * np.abs(o_ref))
    assert excess.max() <= 0, f"{what} O max-abs {err.max():.3e} (above 1e-2 + 2^-8|O| by {excess.max():.3e})"
    assert err.mean() <= O_MEAN_ABS, f"{what} O mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_lse(lse_gpu, lse_ref, what=""):
    g = lse_gpu.double().cpu().numpy() if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    err = np.abs(g - lse_ref)
    assert np.isfinite(err).all(), f"{what} LSE has non-finite values"
    assert err.max() <= LSE_MAX_ABS, f"{what} LSE max-abs {err.max():.3e}"
    return float(err.max())


def check_grad(g_gpu, g_ref, name, what=""):
    g = to_f64(g_gpu) if isinstance(g_gpu, torch.Tensor) else g_gpu
    err = np.abs(g - g_ref)
    bound = GRAD_REL * np.abs(g_ref).max()
    assert np.isfinite(err).all(), f"{what} {name} has non-finite values"
    assert err.max() <= bound, f"{what} {name} max-abs {err.max():.3e} > {bound:.3e}"
    return float(err.max() / max(np.abs(g_ref).max(), 1e-30))


def gpu_inputs(B, H, N, d, seed, dist="normal", with_do=True):
    cpu = make_inputs(B, H, N, d, seed, dist, with_do)
    dev = torch.device("cuda:0")
    return cpu, tuple(None if t is None else t.to(dev) for t in cpu)


def assert_device_ok():
    torch.cuda.synchronize()
    st = binding.device_status(clear=True)
    assert st == binding.FATTN_OK, f"device status {st}: {binding.status_string(st)}"
