"""Helpers shared by the GPU parity tests (data movement and error metrics only)."""
import functools

import numpy as np
import torch

import oracle
from gated_linear_attention_fwd_b200 import inputs

TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(a, dtype="f32"):
    """numpy (bf16-exact values for bf16) -> contiguous CUDA tensor of that storage type."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(TORCH[dtype]).contiguous()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    """max |got - ref| / rms(ref)  (the acceptance metric of the parity tests)."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / rms) if ref.size else 0.0


def tol(dtype):
    """Acceptance bound on max|d|/rms(ref): 1e-4 for fp32 inputs, 1e-2 for bf16 inputs."""
    return 1e-4 if dtype == "f32" else 1e-2


@functools.lru_cache(maxsize=64)
def workload_inputs(index):
    return inputs.make_inputs(inputs.WORKLOADS[index])


@functools.lru_cache(maxsize=64)
def oracle_fwd(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    return oracle.gla_fwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, w.grid_h, w.grid_w, mode)


@functools.lru_cache(maxsize=64)
def oracle_bwd(index, mode):
    w = inputs.WORKLOADS[index]
    x = workload_inputs(index)
    return oracle.gla_bwd(x["q"], x["k"], x["v"], x["z"], w.inv_tau, x["dO"], w.grid_h, w.grid_w, mode)
