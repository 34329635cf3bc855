"""gsa_decode_noalloc: the decode step for callers that cannot allocate
device memory (a plugin or FFI host that only passes input/output pointers,
or a latency-critical caller that must not call cudaMalloc).  It uses the
library's built-in scratch array instead of a caller workspace, so its
results must equal gsa_decode's with a caller-allocated workspace.

Runs last (file name) so that a failure here never hides another test; it
passes both alone in a fresh process and after the rest of the suite.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _decode_both(G, W, cfg, seed):
    x = W.decode_inputs(cfg, device="cuda", own_len=5, seed=seed)
    B, hq, d = x["q"].shape
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, x["gist_k"].shape[2], x["raw_k"].shape[2], cfg.topk,
                       cfg.exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    ref_out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    ref_sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                 ref_out, None, ref_sel, None, ws)
    out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device="cuda")
    sel = torch.full((B, hq, cfg.topk), -5, dtype=torch.int32, device="cuda")
    G.gsa_decode_noalloc(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                         out, None, sel, None)
    torch.cuda.synchronize()
    return ref_out, ref_sel, out, sel, desc, x


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W

    cfg = W.scaled(W.LLAMA_8X, batch=4, context=1024 * 8)
    for call, seed in enumerate((101, 202)):  # two calls in a row, different inputs
        ref_out, ref_sel, out, sel, _, _ = _decode_both(G, W, cfg, seed)
        assert torch.isfinite(out).all(), f"call {call}: output not written"
        err = (out - ref_out).abs().max().item()
        assert err <= 2e-3, f"call {call}: max abs err {err}"
        assert torch.equal(torch.sort(sel, -1).values, torch.sort(ref_sel, -1).values), f"call {call}: selection"


def test_noalloc_rejects_problems_beyond_its_scratch():
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G

    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(4, dtype=torch.int32, device="cuda")
    o = torch.zeros(64, dtype=torch.float32, device="cuda")
    big = G.make_desc(16, 32, 8, 64, 8, 1 << 20, (1 << 20) * 8, 64, False, 0.0, G.GSA_BF16, G.GSA_F32)
    assert G.gsa_workspace_bytes(big, G.GSA_OP_DECODE) > (32 << 20)
    with pytest.raises(G.GsaError) as e:
        G.gsa_decode_noalloc(big, t, t, t, t, t, i, i, o)
    assert e.value.status == G.GSA_ERR_WORKSPACE
