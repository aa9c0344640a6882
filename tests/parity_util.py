"""Helpers shared by the GPU parity tests: move seeded inputs to the GPU, run the
oracle on the same bytes, and compare with the stated tolerances."""
import json
import os

import numpy as np

import oracle
from recurrent_state_memory_b200 import inputs as I

# Parity tolerances:
#   o:   max|o - o_ref| / max|o_ref| <= 1e-4 (fp32 mode), <= 2e-2 (bf16 inputs)
#   S_T: ||S_T - S_ref||_F / ||S_ref||_F <= 1e-2
TOL_O = {"f32": 1e-4, "bf16": 2e-2}
TOL_S = 1e-2


def to_torch(a, device):
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def run_gpu_fwd(p: I.FwdInputs, algo="auto", device="cuda", S0_override=None, want_state=True):
    import torch
    from recurrent_state_memory_b200 import gdr
    t = {key: to_torch(getattr(p, key), device) for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    if S0_override is not None:
        t["S0"] = S0_override
    o, S_T = gdr.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"],
                           gate_mode=p.gate_mode, scale=p.scale, algo=algo, want_state=want_state)
    torch.cuda.synchronize()
    return o, S_T


def o_to_f64(o):
    import torch
    return o.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def oracle_fwd(p: I.FwdInputs):
    return oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                          p.widened("beta"), p.widened("theta"), p.widened("S0"),
                          gate_mode=p.gate_mode, scale=p.scale)


# Every error the GPU tests compute is recorded here, keyed by the running test, so that the
# margin to each tolerance is visible (printed at the end of the run by conftest.py, and
# written as JSON to the file named by GDR_PARITY_LOG when that variable is set).
MARGINS = {}


def _record(kind, value):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    ent = MARGINS.setdefault(test, {})
    ent[kind] = max(ent.get(kind, 0.0), value)


def write_margins(path):
    with open(path, "w") as f:
        json.dump(MARGINS, f, indent=1, sort_keys=True)


def max_rel(a, ref):
    e = float(np.max(np.abs(a - ref)) / max(np.max(np.abs(ref)), 1e-30))
    _record("max_rel", e)
    return e


def rel_l2(a, ref):
    e = float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-30))
    _record("rel_l2", e)
    return e


def assert_fwd_parity(p: I.FwdInputs, o_gpu, S_gpu, o_ref, S_ref, tol_o=None, tol_s=None):
    tol_o = TOL_O[p.dtype] if tol_o is None else tol_o
    tol_s = TOL_S if tol_s is None else tol_s
    og = o_to_f64(o_gpu)
    assert np.all(np.isfinite(og)), "non-finite output"
    eo = max_rel(og, o_ref)
    assert eo <= tol_o, f"o max-rel error {eo:.3e} > {tol_o:.1e}"
    if S_ref is not None and S_gpu is not None:
        es = rel_l2(S_gpu.detach().cpu().numpy().astype(np.float64), S_ref)
        assert es <= tol_s, f"S_T rel-L2 error {es:.3e} > {tol_s:.1e}"
    return eo
