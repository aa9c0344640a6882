"""The C-ABI library: it loads, exports every entry point include/gdr.h declares,
and rejects bad arguments before launching anything (no GPU needed)."""
import ctypes

import pytest

from recurrent_state_memory_b200 import build as gdr_build


@pytest.fixture(scope="module")
def G():
    gdr_build.build()
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    return gdr


def test_exports_every_declared_symbol(G):
    names = G.header_symbols()
    assert {"gdr_chunk_fwd", "gdr_decode_step", "gdr_query_device_status",
            "gdr_chunk_fwd_workspace_bytes", "gdr_status_string", "gdr_abi_version",
            "gdr_last_error_detail"} <= set(names)
    for n in names:
        assert hasattr(G.lib(), n), n


def test_status_strings(G):
    assert G.status_string(0) == "GDR_OK"
    assert G.status_string(4) == "GDR_ERR_TIMEOUT"
    assert G.status_string(6) == "GDR_ERR_RANGE"
    assert G.status_string(99) == "GDR_ERR_UNKNOWN"


def _call_fwd(G, desc, ptrs=None, ws=None, ws_bytes=0):
    p = ptrs or {}
    get = lambda n: ctypes.c_void_p(p[n]) if n in p else None
    return G.lib().gdr_chunk_fwd(ctypes.byref(desc) if desc is not None else None,
                                 get("q"), get("k"), get("v"), get("g"), get("beta"), get("theta"),
                                 get("S0"), get("o"), get("S_T"), ws, ws_bytes, None)


FAKE = {n: 0x10000 * (i + 1) for i, n in enumerate(["q", "k", "v", "g", "beta", "o", "S_T"])}


def _desc(G, **kw):
    import torch
    base = dict(B=1, H=2, T=128, dk=64, dv=64, qkv_dtype=torch.bfloat16, out_dtype=torch.bfloat16)
    base.update(kw)
    return G.fwd_desc(**base)


def test_rejects_bad_arguments_without_launching(G):
    import torch
    L = G.lib()
    assert L.gdr_chunk_fwd(None, *([None] * 10), 0, None) == G.GDR_ERR_INVALID_ARG
    assert _call_fwd(G, _desc(G, dk=48), FAKE) == G.GDR_ERR_UNSUPPORTED
    assert _call_fwd(G, _desc(G, chunk=32), FAKE) == G.GDR_ERR_UNSUPPORTED
    assert _call_fwd(G, _desc(G, B=-1), FAKE) == G.GDR_ERR_INVALID_ARG
    d = _desc(G)
    d.gate_mode = 7
    assert _call_fwd(G, d, FAKE) == G.GDR_ERR_INVALID_ARG
    d = _desc(G)
    d.qkv_dtype = 5
    assert _call_fwd(G, d, FAKE) == G.GDR_ERR_INVALID_ARG
    missing = dict(FAKE)
    del missing["q"]
    assert _call_fwd(G, _desc(G), missing) == G.GDR_ERR_INVALID_ARG
    assert b"required" in L.gdr_last_error_detail()
    misaligned = dict(FAKE, k=FAKE["k"] + 8)
    assert _call_fwd(G, _desc(G), misaligned) == G.GDR_ERR_INVALID_ARG
    assert b"aligned" in L.gdr_last_error_detail()
    assert _call_fwd(G, _desc(G), dict(FAKE, theta=0x900000)) == G.GDR_ERR_INVALID_ARG
    assert _call_fwd(G, _desc(G, rotation=True), FAKE) == G.GDR_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(G):
    assert _call_fwd(G, _desc(G, B=0), {}) == G.GDR_OK
    assert _call_fwd(G, _desc(G, H=0), {}) == G.GDR_OK


def test_decode_rejects_bad_arguments(G):
    import torch
    L = G.lib()
    d = G.DecDesc(4, 2, 128, 128, 1, 1, 1, 0, 1.0)
    assert L.gdr_decode_step(None, *([None] * 8), None) == G.GDR_ERR_INVALID_ARG
    assert L.gdr_decode_step(ctypes.byref(d), *([None] * 8), None) == G.GDR_ERR_INVALID_ARG
    d.dk = 96
    assert L.gdr_decode_step(ctypes.byref(d), *([None] * 8), None) == G.GDR_ERR_UNSUPPORTED
    d0 = G.DecDesc(0, 2, 128, 128, 1, 1, 1, 0, 1.0)
    assert L.gdr_decode_step(ctypes.byref(d0), *([None] * 8), None) == G.GDR_OK


def test_workspace_query(G):
    assert G.workspace_bytes(_desc(G)) >= 0
    assert G.workspace_bytes(_desc(G, dk=48)) == 0


def test_untied_entry_points_check_the_write_strength(G):
    """gdr_chunk_fwd_untied / gdr_decode_step_untied take a write strength w; a misaligned
    w is rejected before any launch, and the tied calls are the untied ones with w = NULL."""
    L = G.lib()
    d = _desc(G)
    get = lambda n: ctypes.c_void_p(FAKE[n])
    st = L.gdr_chunk_fwd_untied(ctypes.byref(d), get("q"), get("k"), get("v"), get("g"), get("beta"),
                                ctypes.c_void_p(0x10004), None, None, get("o"), get("S_T"), None, 0, None)
    assert st == G.GDR_ERR_INVALID_ARG
    import torch
    dd = G.DecDesc(2, 2, 64, 64, 1, 1, 1, 0, 1.0)
    st = L.gdr_decode_step_untied(ctypes.byref(dd), get("q"), get("k"), get("v"), get("g"), get("beta"),
                                  ctypes.c_void_p(0x10004), None, get("S_T"), get("o"), None)
    assert st == G.GDR_ERR_INVALID_ARG


def test_extended_entry_point_checks_the_chunk_mean_output(G):
    """gdr_chunk_fwd_ex adds the chunk-mean output; a misaligned chunk_mean is rejected
    before any launch, as is a misaligned w."""
    L = G.lib()
    d = _desc(G)
    get = lambda n: ctypes.c_void_p(FAKE[n])
    st = L.gdr_chunk_fwd_ex(ctypes.byref(d), get("q"), get("k"), get("v"), get("g"), get("beta"),
                            None, None, None, get("o"), get("S_T"), ctypes.c_void_p(0x10004), None, 0, None)
    assert st == G.GDR_ERR_INVALID_ARG
    assert b"aligned" in L.gdr_last_error_detail()
    st = L.gdr_chunk_fwd_ex(ctypes.byref(d), get("q"), get("k"), get("v"), get("g"), get("beta"),
                            ctypes.c_void_p(0x10004), None, None, get("o"), get("S_T"), get("S_T"), None, 0, None)
    assert st == G.GDR_ERR_INVALID_ARG


def test_host_entry_workspace_and_argument_checks(G):
    """gdr_chunk_fwd_host: the workspace holds two slots of one batch slice's inputs and
    outputs (more with the optional tensors); a short workspace and a missing theta are
    rejected before anything is queued."""
    L = G.lib()
    d = _desc(G, B=2, T=130)             # H=2 dk=dv=64 bf16: two slices of one entry
    base = G.host_workspace_bytes(d)
    per_slice = 130 * 2 * (3 * 64 * 2 + 64 * 4 + 4 + 64 * 2)
    assert base >= 2 * per_slice
    assert G.host_workspace_bytes(d, w=True, S0=True, S_T=True, chunk_mean=True) > base
    get = lambda n: ctypes.c_void_p(FAKE[n])
    args = [get("q"), get("k"), get("v"), get("g"), get("beta"), None, None, None, get("o"), None, None]
    st = L.gdr_chunk_fwd_host(ctypes.byref(d), *args, ctypes.c_void_p(0x100000), base - 1, None)
    assert st == G.GDR_ERR_WORKSPACE
    d.rotation = 1
    st = L.gdr_chunk_fwd_host(ctypes.byref(d), *args, ctypes.c_void_p(0x100000), 1 << 40, None)
    assert st == G.GDR_ERR_INVALID_ARG


def test_auto_resolution_and_workspace_sizes_without_a_device(G):
    """With no device visible the library assumes a B200's 148 SMs.  AUTO's choice follows the
    rules gdr.h states: the fused kernel for a single chunk; the sequence-parallel form for one
    head with a long sequence; split when 2 B*H <= SMs and T > 64; whole fused waves plus a split
    remainder when B*H > SMs and the remainder fits that rule; fused otherwise; the CUDA-core
    kernel for other shapes.  The split workspace is B*H*8 slots of 76,288 bytes plus 36 bytes of
    flags per head and one task counter; the chains kernel's is nc rings of 8 slots of 91,136
    bytes plus 36 bytes of flags and one counter, with 1 <= nc <= min(B*H, 74)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("the 148-SM assumption holds only where no device is visible")
    bf = torch.bfloat16
    d = lambda B, H, T, dk=128, **kw: G.fwd_desc(B, H, T, dk, dk, bf, bf, **kw)
    split = lambda nh: nh * 8 * 76288 + (nh * 8 + nh + 1) * 4
    assert G.resolved_algo(d(4, 16, 4096)) == "tcgen05_split" and G.workspace_bytes(d(4, 16, 4096)) == split(64)
    assert G.resolved_algo(d(2, 37, 4096)) == "tcgen05_split"            # 74 heads: exactly half
    assert G.resolved_algo(d(1, 75, 4096)) == "tcgen05"                  # 75 heads: more than half
    assert G.resolved_algo(d(4, 16, 64)) == "tcgen05"                    # a single chunk
    assert G.resolved_algo(d(4, 16, 65)) == "tcgen05_split"              # two chunks
    assert G.resolved_algo(d(16, 12, 4096)) == "tcgen05_waves"           # 192 = 148 + 44
    assert G.workspace_bytes(d(16, 12, 4096)) == split(44)
    assert G.resolved_algo(d(2, 118, 4096)) == "tcgen05"                 # 236 = 148 + 88: 88 > 74
    assert G.workspace_bytes(d(2, 118, 4096)) == 0
    # one head with a long sequence: its chain alone would be the bound, so the sequence is cut
    # into segments (on the chains kernel); the workspace then also holds y (fp32 per token)
    assert G.resolved_algo(d(1, 1, 4096)) == "tcgen05_segments"
    assert G.workspace_bytes(d(1, 1, 4096)) >= 4096 * 128 * 4
    # the chains kernel on request, for any number of heads
    per_chain = 8 * 91136 + 9 * 4
    for B, H in ((4, 16), (2, 37), (1, 75), (16, 12), (2, 118)):
        desc = d(B, H, 4096, algo="tcgen05_chains")
        assert G.resolved_algo(desc) == "tcgen05_chains"
        n, rem = divmod(G.workspace_bytes(desc) - 4, per_chain)
        assert rem == 0 and 1 <= n <= min(B * H, 74)
    assert G.resolved_algo(d(4, 16, 4096, dk=64)) == "simt"
    f32 = G.fwd_desc(4, 16, 4096, 128, 128, torch.float32, torch.float32)
    assert G.resolved_algo(f32) == "simt" and G.workspace_bytes(f32) == 0


def test_qk_l2norm_flag_is_checked(G):
    d = _desc(G)
    d.qk_l2norm = 2
    assert _call_fwd(G, d, FAKE) == G.GDR_ERR_INVALID_ARG
    d.qk_l2norm = 1
    assert G.lib().gdr_chunk_fwd_workspace_bytes(ctypes.byref(d)) == 0     # SIMT shape here


def test_kernel_launch_count_without_a_device(G):
    """The number of kernels a forward call launches: one for the SIMT, fused and split kernels,
    four for the sequence-parallel form with several segments (two split passes, the scan and
    the correction), none for an empty batch."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("the 148-SM assumption holds only where no device is visible")
    bf = torch.bfloat16
    d = lambda B, H, T, dk=128, **kw: G.fwd_desc(B, H, T, dk, dk, bf, bf, **kw)
    assert G.kernel_launches(d(4, 16, 4096)) == 1                      # split
    assert G.kernel_launches(d(4, 16, 64)) == 1                        # fused, one chunk
    assert G.kernel_launches(d(4, 16, 4096, dk=64)) == 1               # SIMT
    assert G.kernel_launches(d(1, 1, 4096)) == 4                       # segments
    assert G.kernel_launches(d(1, 1, 64, algo="tcgen05_segments", segments=2)) == 1   # one segment
    assert G.kernel_launches(d(0, 16, 4096)) == 0
    with pytest.raises(ValueError):
        G.kernel_launches(G.fwd_desc(1, 1, 64, 48, 48, bf, bf))


def test_backward_checks_its_arguments_without_launching(G):
    """gdr_chunk_bwd: the shapes it does not take are refused before any launch, a missing
    output, a w without its dw or a theta that does not match the rotation flag is an argument
    error, and the workspace size follows the layout (per chunk: three coefficients, the start
    state, the end state's gradient; one scratch region per CTA of the parallel passes)."""
    import ctypes
    import torch
    L = G.lib()
    bf = torch.bfloat16
    d = lambda B, H, T, dk=128, dv=128, **kw: G.fwd_desc(B, H, T, dk, dv, bf, bf, **kw)
    call = lambda desc, ptrs, ws=None, wsb=0: L.gdr_chunk_bwd(ctypes.byref(desc), *ptrs, ws, wsb, None)
    fake = ctypes.c_void_p(1 << 20)        # never dereferenced: every call below fails its checks first
    # q, k, v, g, beta, w, theta, S0, dO, dS_T, dq, dk, dv, dg, dbeta, dw, dtheta, dS0
    rot = [fake] * 18
    full = list(rot)
    full[6] = full[16] = None              # no theta / dtheta without rotation
    assert call(d(1, 1, 64, dk=64, dv=128), full) == G.GDR_ERR_UNSUPPORTED
    assert call(d(1, 1, 64, rotation=True), full) == G.GDR_ERR_INVALID_ARG      # rotation without theta
    assert call(d(1, 1, 64), rot) == G.GDR_ERR_INVALID_ARG                      # theta without rotation
    no_dtheta = list(rot)
    no_dtheta[16] = None
    assert call(d(1, 1, 64, rotation=True), no_dtheta) == G.GDR_ERR_INVALID_ARG
    no_dw = list(full)
    no_dw[15] = None
    assert call(d(1, 1, 64), no_dw) == G.GDR_ERR_INVALID_ARG
    no_dq = list(full)
    no_dq[10] = None
    assert call(d(1, 1, 64), no_dq) == G.GDR_ERR_INVALID_ARG
    assert call(d(1, 1, 64), full, None, 0) == G.GDR_ERR_WORKSPACE
    assert call(d(1, 1, 64, rotation=True), rot, None, 0) == G.GDR_ERR_WORKSPACE
    assert call(d(1, 1, 64, qk_l2norm=True), full, None, 0) == G.GDR_ERR_WORKSPACE
    # scratch per CTA: 18 C x d tiles, 7 C x C tiles, 5 per-token and 3 per-key vectors, S0p
    scratch = 64 * 128 * 18 + 64 * 64 * 7 + 64 * 5 + 128 * 3 + 128 * 128
    dd = 128 * 128
    assert G.bwd_workspace_bytes(d(2, 3, 1000)) == 4 * (6 * 16 * 5 * dd + 96 * scratch)
    assert G.bwd_workspace_bytes(d(4, 16, 4096)) == 4 * (64 * 64 * 5 * dd + 148 * scratch)
    assert G.bwd_workspace_bytes(d(4, 16, 4096, rotation=True)) == G.bwd_workspace_bytes(d(4, 16, 4096))
    assert G.bwd_workspace_bytes(d(2, 3, 0)) == 0


def test_default_build_has_no_index_checks(G):
    """The index checks exist only in the debug build (libgdr_debug.so); the default build
    answers -1 without touching a device."""
    assert G.debug_bounds_site() == -1
    assert G.status_string(G.GDR_ERR_BOUNDS) == "GDR_ERR_BOUNDS"


def test_raven_checks_its_arguments_and_plans_segments(G):
    """gdr_raven_fwd: unsupported shapes and types are refused before any launch, missing
    inputs are argument errors, the segment plan covers the SMs with at least 8 chunks of 32
    tokens per segment, and the workspace holds the earlier segments' end states."""
    import torch
    L = G.lib()
    d = lambda B, H, T, dd=128, K=8, **kw: G.raven_desc(B, H, T, dd, K, **kw)
    fake = ctypes.c_void_p(1 << 20)        # never dereferenced
    call = lambda desc, ptrs, ws=None, wsb=0: L.gdr_raven_fwd(ctypes.byref(desc), *ptrs, ws, wsb, None)
    full = [fake] * 10                     # q, k, v, z, g, S0k, S0v, o, Sk_T, Sv_T
    assert call(d(1, 1, 64, dd=32), full) == G.GDR_ERR_UNSUPPORTED
    assert call(d(1, 1, 64, slots=32), full) == G.GDR_ERR_UNSUPPORTED
    assert call(d(1, 1, 64, K=0), full) == G.GDR_ERR_INVALID_ARG
    assert call(d(1, 1, 64, K=17), full) == G.GDR_ERR_INVALID_ARG
    bad = d(1, 1, 64)
    bad.qkv_dtype = 0
    assert call(bad, full) == G.GDR_ERR_UNSUPPORTED
    no_z = list(full)
    no_z[3] = None
    assert call(d(1, 1, 64), no_z) == G.GDR_ERR_INVALID_ARG
    mis = list(full)
    mis[0] = ctypes.c_void_p((1 << 20) + 8)
    assert call(d(1, 1, 64), mis) == G.GDR_ERR_INVALID_ARG
    # 64 heads of 128 chunks: two segments on 148 SMs; one head of 128 chunks: 16 of 8 chunks
    assert G.raven_segments(d(4, 16, 4096)) == 2
    assert G.raven_segments(d(1, 1, 4096)) == 16
    assert G.raven_segments(d(1, 1, 100)) == 1
    assert G.raven_segments(d(1, 1, 100, segments=3)) == 2          # 4 chunks: 2 per segment
    assert G.raven_segments(d(2, 3, 1000, segments=5)) == 5
    # the state units: 64 chunks before the last segment, cut to 16-chunk units (4 x 64 heads
    # = 256 state CTAs, about two waves on 148 SMs)
    # every token's routing record (144 bytes, the total rounded up to 256), then the state units
    route = lambda n: (n * 144 + 255) // 256 * 256
    assert G.raven_workspace_bytes(d(4, 16, 4096)) == route(4 * 4096 * 16) + 4 * 64 * 4 * (2 * 64 * 128 + 64)
    assert G.raven_workspace_bytes(d(1, 1, 4096)) == route(4096) + 4 * 1 * 30 * (2 * 64 * 128 + 64)   # 16 segments of 8, units of 4
    assert G.raven_workspace_bytes(d(1, 1, 100)) == route(100)
    assert G.raven_workspace_bytes(d(1, 1, 0)) == 0
    assert call(d(4, 16, 4096), full, None, 0) == G.GDR_ERR_WORKSPACE
    assert call(d(1, 1, 100), full, None, 0) == G.GDR_ERR_WORKSPACE
    assert G.raven_workspace_bytes(d(1, 1, 64, dd=32)) == 0
