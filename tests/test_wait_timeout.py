"""Failure detection on the GPU without a fault: every wait in the kernels
is bounded and, on expiry, records GSA_DEVERR_TIMEOUT in the status word,
lets the copies it issued land and returns, so the context stays usable.

A variant of the library is built for this test only, with a 50 ms wait
limit and copy barriers that expect 16 bytes more than their copies bring
(a wait that nothing completes).  The top-k kernel's staging wait and the
unfold's per-warp ring waits must then run out; the calls return, the
status reads TIMEOUT, the top-k result is still exact (the row is read from
global memory after the failed wait), and the normal library keeps working
in the same process.

A second variant (50 ms limit) never publishes row 0 in the fused decode's
ready list: the unfold CTA that waits for the last published row must run
out of its wait and report it, every other row must come out exactly as
the normal library computes it, and the list must be left clear for the
next call."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from long_context_gsa_b200 import _abi, build
    build.build_library()
    stall = build.build_variant(build.PKG / "libgsa_stalltest.so",
                                {"GSA_WAIT_LIMIT_NS": "50000000ull", "GSA_TEST_STALL_BYTES": "16u"})
    return _abi.load(), _abi.load(stall)


def _call_with(lib, fn, *args, **kw):
    """Run a binding function against `lib` instead of the default library."""
    from long_context_gsa_b200 import _abi
    saved = _abi._lib
    _abi._lib = lib
    try:
        return fn(*args, **kw)
    finally:
        _abi._lib = saved


def test_stalled_waits_time_out_and_report(libs):
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W
    normal, stall = libs
    cfg = W.scaled(W.LLAMA_8X, batch=2, context=512 * 8)
    x = W.decode_inputs(cfg, device="cuda", own_len=3)
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, cfg.topk, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    scores = torch.empty((B, hq, n_max), dtype=torch.float32, device="cuda")
    ref_sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    G.gsa_score_gists(desc, x["q"], x["gist_k"], x["gist_v"], x["n_gists"], scores, ws)
    G.gsa_topk_select(desc, scores, x["n_gists"], ref_sel, None, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0

    # top-k: the staging copy's barrier never completes; the kernel reads the row directly
    sel = torch.full_like(ref_sel, -9)
    _call_with(stall, G.gsa_topk_select, desc, scores, x["n_gists"], sel, None, ws)
    torch.cuda.synchronize()
    flags = _call_with(stall, G.gsa_workspace_status, ws)
    assert flags & G.GSA_DEVERR_TIMEOUT, f"status {flags:#x}"
    assert torch.equal(sel, ref_sel)

    # unfold: every ring wait runs out; the call returns and reports it
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    _call_with(stall, G.gsa_unfold_attend, desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"],
               x["own_len"], ref_sel, None, G.GSA_PRIOR_GISTS, out, None, ws)
    torch.cuda.synchronize()
    flags = _call_with(stall, G.gsa_workspace_status, ws)
    assert flags & G.GSA_DEVERR_TIMEOUT, f"status {flags:#x}"

    # the context is still usable: the normal library decodes and reports no error
    G.gsa_workspace_init(ws)
    out2 = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    sel2 = torch.empty_like(ref_sel)
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"], out2,
                 None, sel2, None, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    assert torch.equal(torch.sort(sel2, -1).values, torch.sort(ref_sel, -1).values)
    assert torch.isfinite(out2).all()


@pytest.fixture(scope="module")
def skip_lib():
    from long_context_gsa_b200 import _abi, build
    build.build_library()
    return _abi.load(build.build_variant(build.PKG / "libgsa_skiptest.so",
                                         {"GSA_WAIT_LIMIT_NS": "50000000ull", "GSA_TEST_SKIP_PUBLISH": "1"}))


def test_unpublished_row_times_out(skip_lib):
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W
    cfg = W.scaled(W.LLAMA_8X, batch=2, context=512 * 8)
    x = W.decode_inputs(cfg, device="cuda", own_len=5)
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, cfg.topk, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)

    def decode():
        out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device="cuda")
        G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                     out, None, None, None, ws)
        torch.cuda.synchronize()
        return out

    ref = decode()
    assert G.gsa_workspace_status(ws) == 0
    out = _call_with(skip_lib, decode)
    flags = _call_with(skip_lib, G.gsa_workspace_status, ws)
    assert flags & G.GSA_DEVERR_TIMEOUT, f"status {flags:#x}"
    # every row but row 0 was published and unfolded as usual
    assert torch.equal(out.reshape(B * hq, d)[1:], ref.reshape(B * hq, d)[1:])
    # the last unfold CTA cleared the list: the normal library decodes cleanly
    G.gsa_workspace_init(ws)
    assert torch.equal(decode(), ref)
    assert G.gsa_workspace_status(ws) == 0
