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


def _call_noalloc(G, p, t, out_dtype):
    import torch
    dev = t["q"].device
    desc = G.fwd_desc(p.B, p.H, p.T, p.dk, p.dv, t["q"].dtype, out_dtype, p.gate_mode, p.rotation,
                      p.scale, "auto")
    o = torch.empty((p.B, p.T, p.H, p.dv), dtype=out_dtype, device=dev)
    S_T = torch.empty((p.B, p.H, p.dv, p.dk), dtype=torch.float32, device=dev)
    st = G.lib().gdr_chunk_fwd_noalloc(ctypes.byref(desc), G._ptr(t["q"]), G._ptr(t["k"]), G._ptr(t["v"]),
                                       G._ptr(t["g"]), G._ptr(t["beta"]), G._ptr(t["theta"]), G._ptr(t["S0"]),
                                       G._ptr(o), G._ptr(S_T), G._stream_handle(None, dev))
    assert st == G.GDR_OK, G.lib().gdr_last_error_detail().decode()
    return o, S_T


def test_noalloc_matches_workspace_entry_on_consecutive_calls(G):
    import torch
    cases = [dict(B=2, T=333, H=3, seed=71, rotation=True, s0_std=0.2, out=torch.bfloat16),
             dict(B=4, T=200, H=8, seed=72, rotation=False, s0_std=None, out=torch.float32)]
    for cs in cases:                     # two calls in a row, through the shared scratch
        p = I.make_fwd(cs["B"], cs["T"], cs["H"], 128, 128, dtype="bf16", seed=cs["seed"],
                       rotation=cs["rotation"], s0_std=cs["s0_std"])
        t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
        o_ref, S_ref = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"],
                                   gate_mode=p.gate_mode, algo="tcgen05_split", out_dtype=cs["out"])
        o, S = _call_noalloc(G, p, t, cs["out"])
        torch.cuda.synchronize()
        assert G.query_device_status() == G.GDR_OK
        assert U.max_rel(U.o_to_f64(o), U.o_to_f64(o_ref)) <= U.TOL_O["bf16"]
        assert U.rel_l2(S.cpu().numpy(), S_ref.cpu().numpy()) <= U.TOL_S
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)      # the same kernel and inputs


def test_noalloc_rejects_more_heads_than_its_scratch_holds(G):
    import torch
    desc = G.fwd_desc(3, 11, 128, 128, 128, torch.bfloat16, torch.bfloat16)      # 33 heads > 32
    nul = ctypes.c_void_p(0x1000)
    st = G.lib().gdr_chunk_fwd_noalloc(ctypes.byref(desc), nul, nul, nul, nul, nul, None, None, nul, None, None)
    assert st == G.GDR_ERR_UNSUPPORTED
    assert b"scratch limit of 32 heads" in G.lib().gdr_last_error_detail()
