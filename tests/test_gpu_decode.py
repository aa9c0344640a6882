"""GPU parity of the recurrent decode step against the fp64 oracle."""
import numpy as np
import pytest

import oracle
from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    return gdr


def _run_steps(G, d: I.DecodeInputs, steps, device="cuda"):
    import torch
    S = U.to_torch(d.S, device).clone()
    outs = []
    for s in range(steps):
        t = {key: U.to_torch(getattr(d, key)[s], device) for key in ("q", "k", "v", "g", "beta")}
        th = None if d.theta is None else U.to_torch(d.theta[s], device)
        outs.append(G.decode_step(t["q"], t["k"], t["v"], t["g"], t["beta"], S, th,
                                  gate_mode=d.gate_mode, scale=d.scale))
    torch.cuda.synchronize()
    return outs, S


def _oracle_steps(d: I.DecodeInputs, steps):
    S = d.widened("S")
    outs = []
    for s in range(steps):
        o, S = oracle.gdr_decode_step(d.widened("q", s), d.widened("k", s), d.widened("v", s),
                                      d.widened("g", s), d.widened("beta", s), S,
                                      d.widened("theta", s), d.gate_mode, d.scale)
        outs.append(o)
    return outs, S


@pytest.mark.parametrize("dk,dv,dtype,rot", [
    (128, 128, "bf16", False), (128, 128, "bf16", True), (64, 64, "f32", False),
    (32, 32, "f32", True), (32, 128, "f32", False), (128, 64, "f32", True), (64, 32, "bf16", True)])
def test_decode_parity(G, dk, dv, dtype, rot):
    d = I.make_decode(N=5, H=3, dk=dk, dv=dv, steps=4, dtype=dtype, seed=dk + dv, rotation=rot,
                      s_std=0.3)
    outs, S = _run_steps(G, d, 4)
    ref_outs, S_ref = _oracle_steps(d, 4)
    tol = U.TOL_O[dtype]
    for o, r in zip(outs, ref_outs):
        assert U.max_rel(U.o_to_f64(o), r) <= tol
    assert U.rel_l2(S.cpu().numpy(), S_ref) <= (1e-5 if dtype == "f32" else U.TOL_S)


def test_decode_full_size_sampled(G):
    """The decode workload (256 sequences x 16 heads, dk = dv = 128, fp32 state):
    three steps on the GPU, checked against the oracle on a sample of sequences."""
    import torch
    cfg = dict(I.DECODE_CONFIG)
    cfg["steps"] = 3
    d = I.make_decode(**cfg)
    outs, S = _run_steps(G, d, 3)
    pick = [0, 17, 255]
    sub = I.DecodeInputs(len(pick), d.H, d.dk, d.dv, d.dtype, d.gate_mode, d.rotation,
                         d.q[:, pick], d.k[:, pick], d.v[:, pick], d.g[:, pick], d.beta[:, pick],
                         None, d.S[pick], d.scale)
    ref_outs, S_ref = _oracle_steps(sub, 3)
    for o, r in zip(outs, ref_outs):
        assert U.max_rel(U.o_to_f64(o)[pick], r) <= U.TOL_O["bf16"]
    assert U.rel_l2(S[pick].cpu().numpy(), S_ref) <= U.TOL_S
    assert torch.isfinite(S).all()


def test_decode_steps_match_forward(G):
    """T decode steps reproduce the chunk forward over the same T tokens."""
    import torch
    p = I.make_fwd(3, 70, 2, 64, 64, dtype="f32", seed=55, s0_std=0.3, rotation=True)
    o_fwd, S_fwd = U.run_gpu_fwd(p)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    S = t["S0"].clone()
    outs = []
    for s in range(p.T):
        outs.append(G.decode_step(t["q"][:, s].contiguous(), t["k"][:, s].contiguous(),
                                  t["v"][:, s].contiguous(), t["g"][:, s].contiguous(),
                                  t["beta"][:, s].contiguous(), S, t["theta"][:, s].contiguous()))
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, dim=1)
    assert U.max_rel(U.o_to_f64(o_dec), U.o_to_f64(o_fwd)) < 1e-4
    assert U.rel_l2(S.cpu().numpy(), S_fwd.cpu().numpy()) < 1e-4


@pytest.mark.parametrize("dk,rot", [(128, False), (64, True), (32, True)])
def test_decode_untied_parity(G, dk, rot):
    """Separate erase (beta) and write (w) strengths against the fp64 oracle."""
    import torch
    d = I.make_decode(N=5, H=3, dk=dk, dv=dk, steps=3, dtype="bf16", seed=91 + dk, rotation=rot)
    w = I.make_write_strength(93 + dk, (3, 5, 3))
    S = U.to_torch(d.S, "cuda").clone()
    S_ref = d.widened("S")
    for s in range(3):
        t = {key: U.to_torch(getattr(d, key)[s], "cuda") for key in ("q", "k", "v", "g", "beta")}
        th = None if d.theta is None else U.to_torch(d.theta[s], "cuda")
        o = G.decode_step(t["q"], t["k"], t["v"], t["g"], t["beta"], S, th, gate_mode=d.gate_mode,
                          scale=d.scale, w=torch.from_numpy(w[s]).cuda())
        o_ref, S_ref = oracle.gdr_decode_step(d.widened("q", s), d.widened("k", s), d.widened("v", s),
                                              d.widened("g", s), d.widened("beta", s), S_ref,
                                              d.widened("theta", s), d.gate_mode, d.scale,
                                              w=w[s].astype(np.float64))
        torch.cuda.synchronize()
        assert U.max_rel(U.o_to_f64(o), o_ref) <= U.TOL_O["bf16"]
    assert U.rel_l2(S.cpu().numpy(), S_ref) <= U.TOL_S


@pytest.mark.parametrize("dk,rot", [(128, False), (32, True)])
def test_decode_l2norm_prologue_parity(G, dk, rot):
    """q and k stored with per-token norms far from 1, normalised in the kernel."""
    import torch
    d = I.make_decode(N=4, H=3, dk=dk, dv=dk, steps=2, dtype="f32", seed=95 + dk, rotation=rot, scale=0.7)
    f = np.exp(I.normal(96 + dk, "qkscale", (2, 2, 4, 3, 1)) * 0.7).astype(np.float32)
    S = U.to_torch(d.S, "cuda").clone()
    S_ref = d.widened("S")
    for s in range(2):
        qs, ks = (d.q[s] * f[0, s]).astype(np.float32), (d.k[s] * f[1, s]).astype(np.float32)
        t = {key: U.to_torch(getattr(d, key)[s], "cuda") for key in ("v", "g", "beta")}
        th = None if d.theta is None else U.to_torch(d.theta[s], "cuda")
        o = G.decode_step(U.to_torch(qs, "cuda"), U.to_torch(ks, "cuda"), t["v"], t["g"], t["beta"], S, th,
                          gate_mode=d.gate_mode, scale=d.scale, qk_l2norm=True)
        o_ref, S_ref = oracle.gdr_decode_step(qs.astype(np.float64), ks.astype(np.float64), d.widened("v", s),
                                              d.widened("g", s), d.widened("beta", s), S_ref,
                                              d.widened("theta", s), d.gate_mode, d.scale, qk_l2norm=True)
        torch.cuda.synchronize()
        assert U.max_rel(U.o_to_f64(o), o_ref) <= U.TOL_O["f32"]
    assert U.rel_l2(S.cpu().numpy(), S_ref) <= 1e-4
