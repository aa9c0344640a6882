"""GPU parity of the chunk-WY forward against the fp64 oracle (same seeded bytes)."""
import numpy as np
import pytest

import oracle
from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu

ALGOS_ALL = ["simt", "tcgen05", "tcgen05_split", "tcgen05_chains"]
TC_ALGOS = ["tcgen05", "tcgen05_split", "tcgen05_chains"]


def _skip_unsupported(algo, dtype, dk, dv, nh=1):
    if algo.startswith("tcgen05") and not (dtype == "bf16" and dk == 128 and dv == 128):
        pytest.skip("tcgen05 kernels: bf16 q/k/v with dk = dv = 128 only")
    if algo == "tcgen05_split":
        import torch
        if nh >= torch.cuda.get_device_properties(0).multi_processor_count:
            pytest.skip("split kernel: B*H must be below the SM count (the chains kernel takes any number)")


@pytest.fixture(scope="module")
def G():
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    return gdr


@pytest.mark.parametrize("algo", ["simt"])
def test_tiny_fp32_config(G, algo):
    """The tiny fp32 workload: B=1, H=2, T=256, dk=dv=32, chunk 64, seed 0."""
    p = I.make_config("tiny_f32")
    o, S = U.run_gpu_fwd(p, algo)
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref, tol_o=1e-4, tol_s=1e-4)


CASES = [
    # (B, H, T, dk, dv, dtype, rotation, s0, scale)
    (2, 3, 200, 32, 32, "f32", False, True, 1.0),
    (1, 2, 130, 64, 64, "f32", True, True, 0.5),
    (2, 2, 193, 128, 128, "f32", False, False, 1.0),
    (1, 2, 257, 128, 128, "f32", True, True, 1.0),
    (2, 2, 150, 64, 128, "f32", False, True, 1.0),
    (1, 3, 100, 128, 32, "f32", True, False, 2.0),
    (2, 2, 321, 128, 128, "bf16", False, True, 1.0),
    (1, 2, 190, 128, 128, "bf16", True, True, 1.0),
    (1, 2, 64, 128, 128, "bf16", False, False, 1.0),
]


@pytest.mark.parametrize("algo", ALGOS_ALL)
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}T{}k{}v{}_{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "_rot" if c[6] else "", "_s0" if c[7] else ""))
def test_parity_small(G, algo, case):
    B, H, T, dk, dv, dtype, rot, s0, scale = case
    _skip_unsupported(algo, dtype, dk, dv, B * H)
    p = I.make_fwd(B, T, H, dk, dv, dtype=dtype, seed=1000 + T + dk, rotation=rot,
                   s0_std=0.5 if s0 else None, scale=scale)
    o, S = U.run_gpu_fwd(p, algo)
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref, tol_s=1e-4 if dtype == "f32" else U.TOL_S)


@pytest.mark.parametrize("algo", ["simt"])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129])
def test_chunk_edges(G, algo, T):
    p = I.make_fwd(2, T, 2, 64, 64, dtype="f32", seed=77 + T, rotation=(T % 2 == 1), s0_std=0.3)
    o, S = U.run_gpu_fwd(p, algo)
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref, tol_s=1e-4)


def test_logdecay_gate_mode(G):
    """g passed directly (gate_mode LOGDECAY) including g = 0 (no decay) tokens."""
    import torch
    p = I.make_fwd(1, 150, 2, 64, 64, dtype="f32", seed=5, s0_std=0.3)
    g = -np.logaddexp(0.0, p.g.astype(np.float64)).astype(np.float32)
    g[:, ::7] = 0.0
    p.g = g
    p.gate_mode = I.GATE_LOGDECAY
    o, S = U.run_gpu_fwd(p, "auto")
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref, tol_s=1e-4)


def test_empty_sequence_copies_state(G):
    import torch
    p = I.make_fwd(2, 1, 3, 64, 32, dtype="bf16", seed=9, s0_std=0.5)
    S0 = U.to_torch(p.S0, "cuda")
    z = lambda *s: torch.zeros(*s, device="cuda")
    q = torch.zeros((2, 0, 3, 64), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((2, 0, 3, 32), dtype=torch.bfloat16, device="cuda")
    o, S_T = G.chunk_fwd(q, q, v, z(2, 0, 3, 64), z(2, 0, 3), None, S0)
    torch.cuda.synchronize()
    assert o.numel() == 0
    assert torch.equal(S_T, S0)
    o, S_T = G.chunk_fwd(q, q, v, z(2, 0, 3, 64), z(2, 0, 3), None, None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S_T) == 0


def test_split_resume_and_in_place_state(G):
    """fwd(0..T) == fwd(0..t0) then fwd(t0..T) from its final state, with S_T
    written over S0 in place for the second half."""
    import torch
    p = I.make_fwd(2, 300, 2, 128, 128, dtype="f32", seed=21, s0_std=0.3, rotation=True)
    o_full, S_full = U.run_gpu_fwd(p)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    t0 = 100
    sl = lambda x: x[:, :t0].contiguous()
    sr = lambda x: x[:, t0:].contiguous()
    oa, Sa = G.chunk_fwd(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["g"]), sl(t["beta"]), sl(t["theta"]), t["S0"])
    ob, Sb = G.chunk_fwd(sr(t["q"]), sr(t["k"]), sr(t["v"]), sr(t["g"]), sr(t["beta"]), sr(t["theta"]), Sa,
                         S_T=Sa)
    torch.cuda.synchronize()
    assert Sb.data_ptr() == Sa.data_ptr()
    o_cat = torch.cat([oa, ob], dim=1)
    assert U.max_rel(U.o_to_f64(o_cat), U.o_to_f64(o_full)) < 1e-4
    assert U.rel_l2(Sb.cpu().numpy(), S_full.cpu().numpy()) < 1e-4


def test_deterministic(G):
    import torch
    p = I.make_fwd(2, 200, 2, 128, 128, dtype="bf16", seed=31, s0_std=0.1)
    o1, S1 = U.run_gpu_fwd(p)
    o2, S2 = U.run_gpu_fwd(p)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_host_buffers_round_trip(G):
    """Host (CPU) tensors go through the same library call with copies around it."""
    import torch
    p = I.make_fwd(1, 130, 2, 64, 64, dtype="bf16", seed=41, s0_std=0.2)
    t = {key: U.to_torch(getattr(p, key), "cpu") for key in ("q", "k", "v", "g", "beta", "S0")}
    o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], None, t["S0"])
    assert o.device.type == "cpu" and S.device.type == "cpu"
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


@pytest.mark.parametrize("B,T,rot,algo", [(5, 200, True, "auto"), (11, 130, False, "auto"), (3, 100, False, "simt"),
                                          (3, 0, False, "simt")])
def test_host_entry_pipelines_batch_slices(G, B, T, rot, algo):
    """gdr_chunk_fwd_host on page-locked host tensors (separate write strength, initial state,
    chunk means): the batch runs in slices of ceil(B / min(B, 8)) entries, one device call
    each, with the copies of neighbouring slices overlapped.  Every output equals the device
    calls on the same slices bit for bit, and the oracle within tolerance."""
    import torch
    dk = 128 if algo != "simt" else 64
    p = I.make_fwd(B, T, 2, dk, dk, dtype="bf16", seed=1200 + B + T, rotation=rot, s0_std=0.2)
    w = I.make_write_strength(1201 + B, (B, T, 2))
    keys = ("q", "k", "v", "g", "beta", "theta", "S0")
    h = {key: (None if getattr(p, key) is None else U.to_torch(getattr(p, key), "cpu").pin_memory()) for key in keys}
    wh = torch.from_numpy(w).pin_memory()
    o_h, S_h, m_h = G.chunk_fwd(h["q"], h["k"], h["v"], h["g"], h["beta"], h["theta"], h["S0"],
                                gate_mode=p.gate_mode, algo=algo, w=wh, want_chunk_mean=True)
    assert not o_h.is_cuda and S_h.is_pinned()
    assert T == 0 or (o_h.is_pinned() and m_h.is_pinned())     # (an empty tensor has no pinned storage)
    assert G.query_device_status() == G.GDR_OK
    d = {key: (None if val is None else val.cuda()) for key, val in h.items()}
    wd = wh.cuda()
    bs = -(-B // min(B, 8))
    cut = lambda t, sl: None if t is None else t[sl].contiguous()
    for b0 in range(0, B, bs):
        sl = slice(b0, min(B, b0 + bs))
        o_d, S_d, m_d = G.chunk_fwd(cut(d["q"], sl), cut(d["k"], sl), cut(d["v"], sl), cut(d["g"], sl),
                                    cut(d["beta"], sl), cut(d["theta"], sl), cut(d["S0"], sl),
                                    gate_mode=p.gate_mode, algo=algo, w=cut(wd, sl), want_chunk_mean=True)
        torch.cuda.synchronize()
        assert torch.equal(o_h[sl], o_d.cpu()) and torch.equal(S_h[sl], S_d.cpu()) and torch.equal(m_h[sl], m_d.cpu())
    o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                  p.widened("beta"), p.widened("theta"), p.widened("S0"),
                                  gate_mode=p.gate_mode, scale=p.scale, w=w.astype(np.float64))
    if T == 0:
        assert o_h.numel() == 0 and m_h.shape[1] == 0 and torch.equal(S_h, h["S0"])
        return
    U.assert_fwd_parity(p, o_h, S_h, o_ref, S_ref)
    assert U.max_rel(m_h.numpy().astype(np.float64), oracle.chunk_means(o_ref, 64)) <= U.TOL_O["bf16"]


FULL = ["b4_h16_t4096_d128", "b16_h12_t4096_d128_slow_s0", "b2_h16_t8192_d128_rot"]


@pytest.mark.parametrize("algo", ALGOS_ALL + ["auto"])
@pytest.mark.parametrize("name", FULL)
def test_full_size_configs_sampled(G, algo, name):
    """Full-size workloads in the benchmark's launch configuration; the oracle
    recomputes a sample of whole heads (every token of each sampled head)."""
    cfg = I.FWD_CONFIGS[name]
    _skip_unsupported(algo, cfg["dtype"], cfg["dk"], cfg["dv"], cfg["B"] * cfg["H"])
    p = I.make_config(name)
    o, S = U.run_gpu_fwd(p, algo)
    rng = np.random.default_rng(0)
    heads = [(int(b), int(h)) for b, h in zip(rng.integers(0, p.B, 4), rng.integers(0, p.H, 4))]
    heads += [(0, 0), (p.B - 1, p.H - 1)]
    og = o
    for (b, h) in heads:
        ps = p.head_slice(b, h)
        o_ref, S_ref = U.oracle_fwd(ps)
        o_bh = og[b:b + 1, :, h:h + 1]
        S_bh = S[b:b + 1, h:h + 1]
        U.assert_fwd_parity(ps, o_bh, S_bh, o_ref, S_ref)
    import torch
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()


TC_CASES = [
    # (B, H, T, rotation, s0, out_dtype, gate_mode, scale)
    (1, 2, 1, False, True, "bf16", 1, 1.0),
    (1, 2, 31, True, False, "bf16", 1, 1.0),
    (2, 1, 32, False, True, "f32", 1, 1.0),
    (1, 3, 63, False, False, "bf16", 1, 0.75),
    (2, 2, 64, True, True, "f32", 1, 1.0),
    (1, 2, 65, False, True, "bf16", 0, 1.0),
    (2, 3, 200, True, True, "bf16", 0, 1.0),
    (3, 2, 511, False, True, "f32", 1, 1.0),
]


@pytest.mark.parametrize("algo", TC_ALGOS)
@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "B{}H{}T{}{}{}_{}_g{}".format(
    c[0], c[1], c[2], "_rot" if c[3] else "", "_s0" if c[4] else "", c[5], c[6]))
def test_tcgen05_parity(G, case, algo):
    """The tensor-core kernel against the oracle: ragged tails, rotation, initial state,
    both output dtypes and both gate modes."""
    import torch
    B, H, T, rot, s0, odt, gm, scale = case
    p = I.make_fwd(B, T, H, 128, 128, dtype="bf16", seed=500 + T + 7 * B, rotation=rot,
                   s0_std=0.3 if s0 else None, scale=scale)
    if gm == 0:
        p.g = (-np.logaddexp(0.0, p.g.astype(np.float64))).astype(np.float32)
        p.gate_mode = I.GATE_LOGDECAY
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                       scale=p.scale, algo=algo,
                       out_dtype=torch.float32 if odt == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


def test_auto_picks_tensor_cores_for_bf16_d128(G):
    import torch
    d = G.fwd_desc(1, 1, 64, 128, 128, torch.bfloat16, torch.bfloat16)
    assert G.resolved_algo(d) == "tcgen05"                    # a single chunk: fused
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for B, H, T in ((2, 16, 8192), (4, 16, 4096), (1, 1, 65)):
        d = G.fwd_desc(B, H, T, 128, 128, torch.bfloat16, torch.bfloat16)
        expect = "tcgen05_split" if 2 * B * H <= sms else "tcgen05"   # chains + prep workers
        assert G.resolved_algo(d) == expect
        if expect == "tcgen05_split":
            assert G.workspace_bytes(d) >= B * H * 8 * 76288
    d = G.fwd_desc(16, 12, 4096, 128, 128, torch.bfloat16, torch.bfloat16)
    rem = (16 * 12) % sms if 16 * 12 > sms else 0
    expect = "tcgen05_waves" if 0 < rem and 2 * rem <= sms else "tcgen05"   # many heads
    assert G.resolved_algo(d) == expect
    d = G.fwd_desc(1, 1, 64, 64, 64, torch.bfloat16, torch.bfloat16)
    assert G.resolved_algo(d) == "simt"
    d = G.fwd_desc(1, 1, 64, 128, 128, torch.float32, torch.float32)
    assert G.resolved_algo(d) == "simt"


@pytest.mark.parametrize("rotation", [False, True])
@pytest.mark.parametrize("algo,B,H", [("tcgen05_split", 4, 13), ("tcgen05_chains", 4, 13),
                                      ("tcgen05_chains", 2, 100)])
def test_split_many_heads_parity(G, rotation, algo, B, H):
    """52 heads (one chain each, both split kernels) and 200 heads (more than the SMs: each of
    the chains kernel's chains runs several heads one after another, in waves); six chunks with a
    ragged tail, initial state, against the oracle on every head."""
    B_, T = B, 330
    p = I.make_fwd(B_, T, H, 128, 128, dtype="bf16", seed=77 + int(rotation) + H, s0_std=0.2, rotation=rotation)
    o, S = U.run_gpu_fwd(p, algo)
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


@pytest.mark.parametrize("rotation", [False, True])
def test_split_agrees_with_fused(G, rotation):
    """The split kernel feeds the fp32 E^T to its state MMA as tf32, the fused one rounds it
    to bf16 first: the same result up to rounding."""
    p = I.make_fwd(2, 700, 3, 128, 128, dtype="bf16", seed=61, s0_std=0.2, rotation=rotation)
    o1, S1 = U.run_gpu_fwd(p, "tcgen05")
    o2, S2 = U.run_gpu_fwd(p, "tcgen05_split")
    assert U.max_rel(U.o_to_f64(o2), U.o_to_f64(o1)) <= U.TOL_O["bf16"]
    assert U.rel_l2(S2.cpu().numpy(), S1.cpu().numpy()) <= U.TOL_S


UNTIED_CASES = [
    # (algo, dtype, B, H, T, rotation, s0)
    ("simt", "f32", 1, 2, 133, False, True),
    ("simt", "bf16", 1, 2, 200, True, False),
    ("tcgen05", "bf16", 2, 2, 333, False, True),
    ("tcgen05", "bf16", 1, 3, 200, True, True),
    ("tcgen05_split", "bf16", 2, 3, 333, False, True),
    ("tcgen05_split", "bf16", 2, 2, 450, True, True),
]


@pytest.mark.parametrize("case", UNTIED_CASES, ids=lambda c: "{}_{}_B{}H{}T{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "_rot" if c[5] else "", "_s0" if c[6] else ""))
def test_untied_parity(G, case):
    """Separate erase (beta) and write (w) strengths: every kernel against the fp64 oracle."""
    import torch
    algo, dtype, B, H, T, rot, s0 = case
    dk = 128 if algo != "simt" else 64
    p = I.make_fwd(B, T, H, dk, dk, dtype=dtype, seed=700 + T, rotation=rot, s0_std=0.2 if s0 else None)
    w = I.make_write_strength(701 + T, (B, T, H))
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                       algo=algo, w=torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                  p.widened("beta"), p.widened("theta"), p.widened("S0"),
                                  gate_mode=p.gate_mode, scale=p.scale, w=w.astype(np.float64))
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)
    # and it is not the tied result
    o_t, _ = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                         algo=algo)
    torch.cuda.synchronize()
    assert U.max_rel(U.o_to_f64(o_t), o_ref) > 10 * U.TOL_O[dtype]


@pytest.mark.parametrize("B,rotation", [(1, False), (2, True)])
def test_waves_split_remainder_parity(G, B, rotation):
    """More heads than SMs: whole waves on the fused kernel, the remainder on the split
    kernel (heads offset into the batch), every head against the oracle."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    nh = sms + 12 + (B - 1) * 2                       # a remainder of 12-14 heads
    H = nh // B
    p = I.make_fwd(B, 130, H, 128, 128, dtype="bf16", seed=801 + B, rotation=rotation, s0_std=0.2)
    o, S = U.run_gpu_fwd(p, "tcgen05_waves")
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


CMEAN_CASES = [
    # (algo, dtype, B, H, T, rotation, s0, untied)
    ("simt", "f32", 1, 2, 150, False, True, False),
    ("simt", "bf16", 1, 2, 64, True, False, True),
    ("tcgen05", "bf16", 2, 2, 257, False, True, False),
    ("tcgen05", "bf16", 1, 3, 100, True, True, True),
    ("tcgen05_split", "bf16", 2, 3, 333, False, True, True),
    ("tcgen05_split", "bf16", 1, 2, 200, True, False, False),
]


@pytest.mark.parametrize("case", CMEAN_CASES, ids=lambda c: "{}_{}_B{}H{}T{}{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "_rot" if c[5] else "", "_s0" if c[6] else "", "_untied" if c[7] else ""))
def test_chunk_mean_parity(G, case):
    """The chunk means of o (the extended call's second output, the content signal of the
    content-aware erase) against the oracle's chunk means of its fp64 o; ragged last chunks,
    rotation, initial state, with and without a separate write strength."""
    import torch
    algo, dtype, B, H, T, rot, s0, untied = case
    dk = 128 if algo != "simt" else 64
    p = I.make_fwd(B, T, H, dk, dk, dtype=dtype, seed=1000 + T, rotation=rot, s0_std=0.2 if s0 else None)
    w = I.make_write_strength(1001 + T, (B, T, H)) if untied else None
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    o, S, m = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                          algo=algo, w=None if w is None else torch.from_numpy(w).cuda(), want_chunk_mean=True)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                  p.widened("beta"), p.widened("theta"), p.widened("S0"),
                                  gate_mode=p.gate_mode, scale=p.scale,
                                  w=None if w is None else w.astype(np.float64))
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)
    m_ref = oracle.chunk_means(o_ref, 64)
    assert tuple(m.shape) == m_ref.shape
    assert U.max_rel(m.cpu().numpy().astype(np.float64), m_ref) <= U.TOL_O[dtype]


def test_chunk_mean_with_waves_and_on_host_buffers(G):
    """More heads than SMs (fused waves plus a split remainder, heads offset into the batch)
    with the chunk means requested; then the same call on host tensors returns the same
    three outputs."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, H, T = 1, sms + 13, 130
    p = I.make_fwd(B, T, H, 128, 128, dtype="bf16", seed=1100, s0_std=0.2)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "S0")}
    o, S, m = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], None, t["S0"], gate_mode=p.gate_mode,
                          want_chunk_mean=True, algo="tcgen05_waves")
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)
    assert U.max_rel(m.cpu().numpy().astype(np.float64), oracle.chunk_means(o_ref, 64)) <= U.TOL_O["bf16"]
    h = {key: val.cpu() for key, val in t.items()}
    o_h, S_h, m_h = G.chunk_fwd(h["q"], h["k"], h["v"], h["g"], h["beta"], None, h["S0"], gate_mode=p.gate_mode,
                                want_chunk_mean=True, algo="tcgen05_waves")
    assert not o_h.is_cuda and torch.equal(o_h, o.cpu()) and torch.equal(S_h, S.cpu()) and torch.equal(m_h, m.cpu())


L2NORM_CASES = [
    # (algo, dtype, B, H, T, rotation)
    ("simt", "f32", 1, 2, 150, False),
    ("tcgen05", "bf16", 2, 2, 257, True),
    ("tcgen05_split", "bf16", 2, 3, 333, False),
]


@pytest.mark.parametrize("case", L2NORM_CASES, ids=lambda c: "{}_{}_B{}H{}T{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "_rot" if c[5] else ""))
def test_l2norm_prologue_parity(G, case):
    """q and k stored un-normalised (per-token norms in [0.25, 4]), normalised in the kernel:
    against the oracle with its own fp64 normalisation of the same stored values."""
    import torch
    algo, dtype, B, H, T, rot = case
    dk = 128 if algo != "simt" else 64
    p = I.make_fwd(B, T, H, dk, dk, dtype="f32", seed=900 + T, rotation=rot, s0_std=0.2, scale=0.8)
    f = np.exp(I.normal(901 + T, "qkscale", (2, B, T, H, 1)) * 0.5).astype(np.float32)
    q = (p.q * f[0]).astype(np.float32)
    k = (p.k * f[1]).astype(np.float32)
    if dtype == "bf16":
        q, k, v = I.to_bf16_bits(q), I.to_bf16_bits(k), I.to_bf16_bits(p.v)
        p = I.FwdInputs(p.B, p.T, p.H, p.dk, p.dv, p.chunk, "bf16", p.gate_mode, p.rotation, q, k, v,
                        p.g, p.beta, p.theta, p.S0, p.scale)
    else:
        p.q, p.k = q, k
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("q", "k", "v", "g", "beta", "theta", "S0")}
    o, S = G.chunk_fwd(t["q"], t["k"], t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                       scale=p.scale, algo=algo, qk_l2norm=True)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = oracle.gdr_fwd(p.widened("q"), p.widened("k"), p.widened("v"), p.widened("g"),
                                  p.widened("beta"), p.widened("theta"), p.widened("S0"),
                                  gate_mode=p.gate_mode, scale=p.scale, qk_l2norm=True)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


def test_full_size_with_both_optional_features_sampled(G):
    """The bench workload with a separate write strength and the fused L2 normalisation
    together (q and k stored at norms far from 1), AUTO's launch configuration, sampled
    whole heads against the oracle."""
    import torch
    p = I.make_config("b4_h16_t4096_d128")
    w = I.make_write_strength(77, (p.B, p.T, p.H))
    f = np.exp(I.normal(78, "qkscale", (2, p.B, p.T, p.H, 1)) * 0.5).astype(np.float32)
    q32 = U.to_torch(p.q, "cuda").float() * torch.from_numpy(f[0]).cuda()
    k32 = U.to_torch(p.k, "cuda").float() * torch.from_numpy(f[1]).cuda()
    q16, k16 = q32.to(torch.bfloat16), k32.to(torch.bfloat16)
    t = {key: U.to_torch(getattr(p, key), "cuda") for key in ("v", "g", "beta", "theta", "S0")}
    o, S = G.chunk_fwd(q16, k16, t["v"], t["g"], t["beta"], t["theta"], t["S0"], gate_mode=p.gate_mode,
                       scale=p.scale, w=torch.from_numpy(w).cuda(), qk_l2norm=True)
    torch.cuda.synchronize()
    assert G.query_device_status() == G.GDR_OK
    qh, kh = q16.float().cpu().numpy(), k16.float().cpu().numpy()
    for (b, h) in [(0, 0), (1, 7), (p.B - 1, p.H - 1)]:
        ps = p.head_slice(b, h)
        o_ref, S_ref = oracle.gdr_fwd(qh[b:b + 1, :, h:h + 1], kh[b:b + 1, :, h:h + 1], ps.widened("v"),
                                      ps.widened("g"), ps.widened("beta"), ps.widened("theta"), ps.widened("S0"),
                                      gate_mode=p.gate_mode, scale=p.scale, w=w[b:b + 1, :, h:h + 1].astype(np.float64),
                                      qk_l2norm=True)
        U.assert_fwd_parity(ps, o[b:b + 1, :, h:h + 1], S[b:b + 1, h:h + 1], o_ref, S_ref)
