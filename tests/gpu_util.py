"""Helpers for the GPU tests: device upload, calls through the binding, error metric."""
import numpy as np
import torch

import gated_delta_rule_97_b200 as gdn

# Parity bounds: max|diff| / rms(reference) over the compared tensor.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-300))


def dev(x, dtype=torch.float32):
    if x is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda().to(dtype).contiguous()


def io_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def run_prefill(w, x, algo="auto", out_dtype=torch.float32, S0_dev=None):
    dt = io_dtype(w)
    o, ST = gdn.chunk_fwd(dev(x["q"], dt), dev(x["k"], dt), dev(x["v"], dt), dev(x["g"]), dev(x["beta"]),
                          S0_dev if S0_dev is not None else dev(x["S0"]), update=w.update, gate=w.gate,
                          out_dtype=out_dtype, algo=algo)
    torch.cuda.synchronize()
    diag = gdn.device_diag()
    status = gdn.device_status()
    assert status == 0, ("device status", status, "diag", diag)
    return o, ST


def np64(t):
    return t.float().cpu().numpy().astype(np.float64)
