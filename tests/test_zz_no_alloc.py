"""gdr_chunk_fwd_noalloc: the forward for callers that cannot hand the library device
memory.  Examples are hosts whose own allocator owns the whole GPU, and latency paths that must
not call cudaMalloc, which can synchronise the device.

It must give the same output as gdr_chunk_fwd (caller workspace, same split kernel) on the
same inputs, on consecutive calls, although every call reuses the one scratch array built
into the library.  The file is collected last, so a run that stops at the first failure has
already run every other test.
"""
import ctypes

import pytest

from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    return gdr


def _call_noalloc(G, p, t, out_dtype, qk_l2norm=False):
    import torch
    dev = t["q"].device
    desc = G.fwd_desc(p.B, p.H, p.T, p.dk, p.dv, t["q"].dtype, out_dtype, p.gate_mode, p.rotation,
                      p.scale, "auto", qk_l2norm=qk_l2norm)
    o = torch.empty((p.B, p.T, p.H, p.dv), dtype=out_dtype, device=dev)
    S_T = torch.empty((p.B, p.H, p.dv, p.dk), dtype=torch.float32, device=dev)
    st = G.lib().gdr_chunk_fwd_noalloc(ctypes.byref(desc), G._ptr(t["q"]), G._ptr(t["k"]), G._ptr(t["v"]),
                                       G._ptr(t["g"]), G._ptr(t["beta"]), G._ptr(t["theta"]), G._ptr(t["S0"]),
                                       G._ptr(o), G._ptr(S_T), G._stream_handle(None, dev))
    assert st == G.GDR_OK, G.lib().gdr_last_error_detail().decode()
    return o, S_T


# Consecutive calls through the one shared scratch array: a 6-head call, the largest call the
# array holds (32 heads), then smaller calls after it (4 heads with the fused L2
# normalisation, 10 heads with a single chunk), so that flags left behind by a larger call
# meet a later, smaller one; then a call with no tokens at all (S_T = S0).
CASES = [dict(B=2, T=333, H=3, seed=71, rotation=True, s0_std=0.2, out="bf16"),
         dict(B=4, T=200, H=8, seed=72, rotation=False, s0_std=None, out="f32"),
         dict(B=1, T=150, H=4, seed=73, rotation=False, s0_std=0.1, out="bf16", l2=True),
         dict(B=2, T=64, H=5, seed=74, rotation=True, s0_std=None, out="bf16"),
         dict(B=3, T=0, H=2, seed=75, rotation=False, s0_std=0.3, out="f32")]


def test_noalloc_matches_oracle_and_workspace_entry_on_consecutive_calls(G):
    import torch
    import oracle
    for cs in CASES:
        out = torch.bfloat16 if cs["out"] == "bf16" else torch.float32
        l2 = cs.get("l2", False)
        p = I.make_fwd(cs["B"], cs["T"], cs["H"], 128, 128, dtype="bf16", seed=cs["seed"],
                       rotation=cs["rotation"], s0_std=cs["s0_std"])
        t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
        o, S = _call_noalloc(G, p, t, out, qk_l2norm=l2)
        torch.cuda.synchronize()
        assert G.query_device_status() == G.GDR_OK
        o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                      p.widened("beta"), p.widened("theta"), p.widened("S0"),
                                      gate_mode=p.gate_mode, scale=p.scale, qk_l2norm=l2)
        if p.T == 0:
            assert torch.equal(S, t["S0"])                 # no tokens: the state passes through
        else:
            U.assert_fwd_parity(p, o, S, o_ref, S_ref)
        # the workspace entry with the same (split) kernel gives the same bytes
        if p.T > 0:
            o_w, S_w = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"],
                                   gate_mode=p.gate_mode, algo="tcgen05_split", out_dtype=out, qk_l2norm=l2)
            torch.cuda.synchronize()
            assert torch.equal(o, o_w) and torch.equal(S, S_w)


def test_noalloc_rejects_more_heads_than_its_scratch_holds(G):
    import torch
    desc = G.fwd_desc(3, 11, 128, 128, 128, torch.bfloat16, torch.bfloat16)      # 33 heads > 32
    nul = ctypes.c_void_p(0x1000)
    st = G.lib().gdr_chunk_fwd_noalloc(ctypes.byref(desc), nul, nul, nul, nul, nul, None, None, nul, None, None)
    assert st == G.GDR_ERR_UNSUPPORTED
    assert b"scratch limit of 32 heads" in G.lib().gdr_last_error_detail()
