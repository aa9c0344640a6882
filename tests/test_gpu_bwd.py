"""GPU parity of the backward pass (gdr_chunk_bwd) against the fp64 oracle's reverse-mode sweep
of the token recurrence (oracle/backward.py): every input gradient, element by element.

Tolerance: the kernel computes in fp32 (split-tf32 tensor-core products, fp32 elsewhere) on the
same bf16/fp32 input values the oracle widens, so its error is fp32 rounding accumulated along
the chunk chain; each gradient must satisfy max|d - d_ref| / max|d_ref| <= 1e-3."""
import numpy as np
import pytest

from oracle.backward import gdr_bwd
from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu

TOL_BWD = 1e-3


@pytest.fixture(scope="module")
def G():
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    return gdr


BWD_CASES = [
    # (B, H, T, d, dtype, gate_mode, untied w, S0, dO, dS_T, gate recipe, rotation, qk_l2norm)
    (1, 2, 128, 128, "bf16", 1, False, False, True, True, "normal", False, False),
    (2, 1, 100, 64, "f32", 0, False, True, True, False, "normal", False, False),      # ragged, log-decay gates
    (1, 3, 200, 32, "bf16", 1, True, True, True, True, "normal", False, False),       # ragged, separate w
    (1, 1, 64, 128, "f32", 1, False, True, False, True, "normal", False, False),      # only dS_T
    (2, 2, 257, 128, "bf16", 1, False, True, True, True, "normal", False, False),     # one-token tail
    (1, 1, 512, 128, "bf16", 1, False, True, True, True, "slow", False, False),       # slow decay, 8 chunks
    (1, 2, 200, 128, "bf16", 1, False, True, True, True, "normal", True, False),      # rotation, ragged
    (2, 1, 130, 64, "f32", 0, True, True, True, True, "normal", True, False),         # rotation, log-decay, w
    (1, 2, 150, 128, "bf16", 1, False, True, True, True, "normal", False, True),      # qk_l2norm
    (1, 1, 100, 32, "f32", 1, True, True, True, True, "slow", True, True),            # rotation + qk_l2norm
]


def _case_id(c):
    B, H, T, d, dt, gm, w, s0, do, ds, gate, rot, nrm = c
    return f"B{B}H{H}T{T}d{d}_{dt}_g{gm}" + ("_w" if w else "") + ("_s0" if s0 else "") + \
        ("_dO" if do else "") + ("_dS" if ds else "") + ("_slow" if gate == "slow" else "") + \
        ("_rot" if rot else "") + ("_l2" if nrm else "")


def _inputs(case, seed):
    B, H, T, d, dt, gm, untied, s0, with_dO, with_dS, gate, rot, nrm = case
    p = I.make_fwd(B, T, H, d, d, dtype=dt, seed=seed, gate=gate, s0_std=0.3 if s0 else None, rotation=rot)
    if nrm:     # raw q and k of norms far from one (the kernel normalises them)
        for n in ("q", "k"):
            x = I.normal(seed, n + "_raw", (B, T, H, d)).astype(np.float32) * \
                (0.5 + 3.0 * I.uniform(seed, n + "_len", B * T * H).reshape(B, T, H, 1)).astype(np.float32)
            setattr(p, n, I.to_bf16_bits(x) if dt == "bf16" else x)
    g = p.g if gm == 1 else (-np.logaddexp(0.0, p.g.astype(np.float64))).astype(np.float32)   # log-decay values
    w = I.make_write_strength(seed + 1, (B, T, H)) if untied else None
    dO = I.normal(seed, "dO", (B, T, H, d)).astype(np.float32) if with_dO else None
    if dO is not None and dt == "bf16":
        dO = I.to_bf16_bits(dO)
    dS = I.normal(seed, "dS_T", (B, H, d, d), std=0.5).astype(np.float32) if with_dS else None
    return p, g, w, dO, dS


def _widen(a):
    if a is None:
        return None
    return (I.bf16_bits_to_f32(a) if a.dtype == np.uint16 else a).astype(np.float64)


@pytest.mark.parametrize("case", BWD_CASES, ids=_case_id)
def test_backward_parity(G, case):
    import torch
    p, g, w, dO, dS = _inputs(case, 700 + case[2] + case[3])
    gm, rot, nrm = case[5], case[11], case[12]
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "beta", "S0", "theta")}
    gt = U.to_torch(g, "cuda")
    wt, dOt, dSt = U.to_torch(w, "cuda"), U.to_torch(dO, "cuda"), U.to_torch(dS, "cuda")
    grads = G.chunk_bwd(t["q"], t["k"], t["v"], gt, t["beta"], t["S0"], dOt, dSt, gate_mode=gm, w=wt,
                        theta=t["theta"], qk_l2norm=nrm, out_dtype=t["q"].dtype)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    _, _, ref = gdr_bwd(p.widened("q"), p.widened("k"), p.widened("v"), g.astype(np.float64),
                        p.widened("beta"), None if not rot else p.theta.astype(np.float64), p.widened("S0"),
                        _widen(dO), _widen(dS), gate_mode=gm, scale=p.scale,
                        w=None if w is None else w.astype(np.float64), qk_l2norm=nrm)
    names = ["q", "k", "v", "g", "beta", "S0"] + (["w"] if w is not None else []) + (["theta"] if rot else [])
    for n in names:
        got = grads[n].cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"non-finite d{n}"
        e = U.max_rel(got, ref[n])
        assert e <= TOL_BWD, f"d{n}: max-rel error {e:.3e} > {TOL_BWD:.0e}"


def test_backward_without_tokens_passes_the_state_gradient(G):
    import torch
    q = torch.zeros((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((1, 0, 2, 64), dtype=torch.float32, device="cuda")
    beta = torch.zeros((1, 0, 2), dtype=torch.float32, device="cuda")
    dS = torch.from_numpy(I.normal(5, "dS_T", (1, 2, 64, 64)).astype(np.float32)).cuda()
    grads = G.chunk_bwd(q, q, v, g, beta, None, None, dS)
    torch.cuda.synchronize()
    assert torch.equal(grads["S0"], dS)


def test_backward_matches_a_finite_difference_of_the_forward_kernel(G):
    """The backward kernel against the forward kernel itself: the directional derivative of
    <dO, o> + <dS_T, S_T> along a random direction of beta, by central differences of two
    fp32 forward launches, equals <dbeta, direction>."""
    import torch
    B, H, T, d = 1, 2, 130, 64
    p = I.make_fwd(B, T, H, d, d, dtype="f32", seed=771, s0_std=0.2)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "S0")}
    dO = torch.from_numpy(I.normal(772, "dO", (B, T, H, d)).astype(np.float32)).cuda()
    dS = torch.from_numpy(I.normal(773, "dS_T", (B, H, d, d)).astype(np.float32)).cuda()
    dirn = torch.from_numpy(I.normal(774, "dir", (B, T, H)).astype(np.float32)).cuda()
    grads = G.chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], dO, dS)
    h = 1e-3

    def loss(beta):
        o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], beta, None, t["S0"], algo="simt")
        return float((o.double() * dO.double()).sum() + (S.double() * dS.double()).sum())

    fd = (loss(t["beta"] + h * dirn) - loss(t["beta"] - h * dirn)) / (2 * h)
    an = float((grads["beta"].double() * dirn.double()).sum())
    assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), (fd, an)


def test_backward_full_size_sampled_heads(G):
    """The bench workload (B=4 H=16 T=4096 d=128, bf16) with dO and dS_T: every gradient of
    three sampled heads against the oracle's chunked restatement of the reverse sweep
    (oracle/backward.py::chunk_bwd_head, pinned to the token sweep on the CPU)."""
    import torch
    from oracle.backward import chunk_bwd_head
    p = I.make_config("b4_h16_t4096_d128")
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta")}
    dO = I.to_bf16_bits(I.normal(780, "dO", (p.B, p.T, p.H, p.dv)).astype(np.float32))
    dS = I.normal(781, "dS_T", (p.B, p.H, p.dv, p.dk), std=0.5).astype(np.float32)
    grads = G.chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], None, U.to_torch(dO, "cuda"),
                        U.to_torch(dS, "cuda"), gate_mode=p.gate_mode, scale=p.scale, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    dO64 = I.bf16_bits_to_f32(dO).astype(np.float64)
    for (b, h) in ((0, 0), (2, 9), (3, 15)):
        sel = lambda a: a[b, :, h]
        _, _, ref = chunk_bwd_head(sel(p.widened("q")), sel(p.widened("k")), sel(p.widened("v")),
                                   sel(p.widened("g")), sel(p.widened("beta")), None, sel(dO64),
                                   dS[b, h].astype(np.float64), p.gate_mode, p.scale, None)
        for n in ("q", "k", "v", "g", "beta"):
            got = grads[n][b, :, h].cpu().numpy().astype(np.float64)
            e = U.max_rel(got, ref[n])
            assert e <= TOL_BWD, f"d{n} of head ({b},{h}): max-rel error {e:.3e}"
        e = U.max_rel(grads["S0"][b, h].cpu().numpy().astype(np.float64), ref["S0"])
        assert e <= TOL_BWD, f"dS0 of head ({b},{h}): max-rel error {e:.3e}"
