"""The debug build (libgdr_debug.so, -DGDR_BOUNDS_CHECK): every kernel tests the index of each
global-memory access it computes before making it.  On small and ragged shapes through every
kernel (split, waves, segments, fused, CUDA-core forward, decode, backward with and without
rotation and the L2 normalisation, Raven's slot memory) no test fails, and
the outputs equal the default build's (the checks change no arithmetic; the compiler may still
contract a product differently around the added branches, so one rounding step of the output
type is allowed)."""
import os

import numpy as np
import pytest

from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    from recurrent_state_memory_b200 import build, gdr
    default = gdr.LIB_PATH
    dbg = build.LIB_DEBUG
    if not os.path.exists(dbg):
        pytest.fail("libgdr_debug.so is missing: __graft_entry__.build() builds it")
    yield gdr, default, dbg
    gdr.use_library(default)


FWD_CASES = [
    # (B, H, T, d, dtype, algo, rotation, S0, w, chunk mean, segments)
    (2, 3, 333, 128, "bf16", "tcgen05_split", False, True, False, False, 0),
    (1, 2, 200, 128, "bf16", "tcgen05_split", True, True, False, True, 0),
    (3, 50, 130, 128, "bf16", "tcgen05_waves", False, True, True, True, 0),
    (2, 1, 1000, 128, "bf16", "tcgen05_segments", False, True, False, False, 3),
    (1, 3, 777, 128, "bf16", "tcgen05_segments", True, False, False, True, 4),
    (2, 2, 64, 128, "bf16", "tcgen05", False, True, False, False, 0),
    (1, 2, 150, 64, "f32", "simt", False, True, True, True, 0),
    (1, 1, 0, 128, "bf16", "auto", False, True, False, False, 0),
]


def _same(a, b):
    import torch
    if torch.equal(a, b):
        return True
    tol = 8e-3 if a.dtype == torch.bfloat16 else 1e-5
    return U.max_rel(a.double().cpu().numpy(), b.double().cpu().numpy()) <= tol


def _fwd(gdr, case):
    import torch
    B, H, T, d, dt, algo, rot, s0, w, cm, nseg = case
    p = I.make_fwd(B, T, H, d, d, dtype=dt, seed=40 + T, rotation=rot, s0_std=0.2 if s0 else None)
    t = {k: U.to_torch(getattr(p, k), "cuda") for k in ("q", "k", "v", "g", "beta", "theta", "S0")}
    wt = torch.from_numpy(I.make_write_strength(41, (B, T, H))).cuda() if w else None
    out = gdr.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                        algo=algo, w=wt, want_chunk_mean=cm, segments=nseg)
    torch.cuda.synchronize()
    return [None if x is None else x.clone() for x in out]


@pytest.mark.parametrize("case", FWD_CASES, ids=lambda c: f"{c[5]}_B{c[0]}H{c[1]}T{c[2]}d{c[3]}")
def test_debug_build_forward(G, case):
    import torch
    gdr, default, dbg = G
    gdr.use_library(default)
    ref = _fwd(gdr, case)
    gdr.use_library(dbg)
    assert gdr.debug_bounds_site() == 0
    got = _fwd(gdr, case)
    assert gdr.query_device_status() == gdr.GDR_OK
    assert gdr.debug_bounds_site() == 0
    for a, b in zip(got, ref):
        if a is not None:
            assert _same(a, b)


def test_debug_build_raven(G):
    """Raven's two passes (three segments, a ragged tail) on the debug build."""
    import torch
    p = I.make_raven(2, 200, 2, 64, K=4, seed=14, s0_std=0.3)
    t = {n: U.to_torch(getattr(p, n), "cuda") for n in ("q", "k", "v", "z", "g", "S0k", "S0v")}
    res = {}
    for name, path in (("default", G[1]), ("debug", G[2])):
        G[0].use_library(path)
        out = G[0].raven_fwd(t["q"], t["k"], t["v"], t["z"], t["g"], t["S0k"], t["S0v"], topk=p.K, scale=p.scale,
                             segments=3)
        torch.cuda.synchronize()
        assert G[0].query_device_status() == G[0].GDR_OK
        if name == "debug":
            assert G[0].debug_bounds_site() == 0
        res[name] = [x.clone() for x in out]
    for a, b in zip(res["debug"], res["default"]):
        assert _same(a, b)


def test_debug_build_decode_and_backward(G):
    import torch
    gdr, default, dbg = G
    dc = I.make_decode(N=4, H=4, dk=128, dv=128, steps=2, dtype="bf16", seed=9, s_std=0.1)   # 16-byte aligned per step
    p = I.make_fwd(1, 130, 2, 64, 64, dtype="bf16", seed=10, s0_std=0.2)
    pr = I.make_fwd(2, 77, 1, 32, 32, dtype="f32", seed=12, s0_std=0.2, rotation=True)      # rotation, ragged
    dS = torch.from_numpy(I.normal(13, "dS_T", (2, 1, 32, 32)).astype(np.float32)).cuda()
    res = {}
    for name, path in (("default", default), ("debug", dbg)):
        gdr.use_library(path)
        S = U.to_torch(dc.S, "cuda").clone()
        d = {k: U.to_torch(getattr(dc, k), "cuda") for k in ("q", "k", "v", "g", "beta")}
        o = [gdr.decode_step(d["q"][i], d["k"][i], d["v"][i], d["g"][i], d["beta"][i], S, gate_mode=dc.gate_mode)
             for i in range(2)]
        t = {k: U.to_torch(getattr(p, k), "cuda") for k in ("q", "k", "v", "g", "beta", "S0")}
        dO = torch.from_numpy(I.normal(11, "dO", (1, 130, 2, 64)).astype(np.float32)).cuda().to(torch.bfloat16)
        grads = gdr.chunk_bwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], dO, None)
        tr = {k: U.to_torch(getattr(pr, k), "cuda") for k in ("q", "k", "v", "g", "beta", "S0", "theta")}
        grads_r = gdr.chunk_bwd(tr["q"], tr["k"], tr["v"], tr["g"], tr["beta"], tr["S0"], None, dS,
                                theta=tr["theta"], qk_l2norm=True)
        torch.cuda.synchronize()
        assert gdr.query_device_status() == gdr.GDR_OK
        if name == "debug":
            assert gdr.debug_bounds_site() == 0
        res[name] = (S, o, grads, grads_r)
    Sd, od, gd, grd = res["debug"]
    S0_, o0, g0, gr0 = res["default"]
    assert _same(Sd, S0_) and all(_same(a, b) for a, b in zip(od, o0))
    for a, b in ((gd, g0), (grd, gr0)):
        for n, x in b.items():
            if x is not None:
                assert _same(a[n], x)
