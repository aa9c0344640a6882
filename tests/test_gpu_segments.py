"""GPU parity of the sequence-parallel forward (GDR_ALGO_TCGEN05_SEGMENTS) against the fp64
token oracle: each head's sequence is cut into segments that run as separate chains from the
zero state and from the identity, then combined through the exact affine chunk transfer
("Semidirect Fourier Delta Attention" page, "Main contributions")."""
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


SEG_CASES = [
    # (B, H, T, segments, rotation, s0, out dtype)
    (1, 2, 1024, 4, False, False, "bf16"),      # whole segments
    (2, 1, 1000, 3, False, True, "bf16"),       # ragged: 384-token segments, the last one 232
    (1, 3, 777, 4, True, True, "bf16"),         # rotation, ragged tail inside the last chunk
    (1, 1, 4096, 16, True, False, "f32"),       # many segments
    (2, 2, 300, 2, False, True, "f32"),
]


@pytest.mark.parametrize("case", SEG_CASES, ids=lambda c: "B{}H{}T{}_seg{}{}{}_{}".format(
    c[0], c[1], c[2], c[3], "_rot" if c[4] else "", "_s0" if c[5] else "", c[6]))
def test_segments_parity(G, case):
    import torch
    B, H, T, nseg, rot, s0, odt = case
    p = I.make_fwd(B, T, H, 128, 128, dtype="bf16", seed=900 + T + nseg, rotation=rot, s0_std=0.3 if s0 else None)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                       algo="tcgen05_segments", segments=nseg,
                       out_dtype=torch.float32 if odt == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


def test_segments_agree_with_one_chain_per_head(G):
    """The same inputs through the plain split kernel (one chain per head) and through four
    segments: the same o and S_T up to rounding; with the chunk means of o and a separate
    write strength, which the segments carry through (the mean is linear in o)."""
    import torch
    B, H, T = 1, 2, 2048
    p = I.make_fwd(B, T, H, 128, 128, dtype="bf16", seed=951, s0_std=0.2)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    w = torch.from_numpy(I.make_write_strength(952, (B, T, H))).cuda()
    o1, S1, m1 = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], None, t["S0"], gate_mode=p.gate_mode,
                             algo="tcgen05_split", w=w, want_chunk_mean=True)
    o2, S2, m2 = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], None, t["S0"], gate_mode=p.gate_mode,
                             algo="tcgen05_segments", segments=4, w=w, want_chunk_mean=True)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    assert U.max_rel(U.o_to_f64(o2), U.o_to_f64(o1)) <= U.TOL_O["bf16"]
    assert U.rel_l2(S2.cpu().numpy(), S1.cpu().numpy()) <= U.TOL_S
    assert U.max_rel(m2.cpu().numpy().astype(np.float64), m1.cpu().numpy().astype(np.float64)) <= U.TOL_O["bf16"]
    o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                  p.widened("beta"), None, p.widened("S0"), gate_mode=p.gate_mode,
                                  w=w.cpu().numpy().astype(np.float64))
    U.assert_fwd_parity(p, o2, S2, o_ref, S_ref)
    assert U.max_rel(m2.cpu().numpy().astype(np.float64), oracle.chunk_means(o_ref, 64)) <= U.TOL_O["bf16"]
