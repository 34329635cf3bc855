"""Boundary checks that need real device buffers: the binding refuses a
short buffer at any argument position before the library is called, so no
kernel ever reads or writes past a caller's allocation."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G_
    return G_


def test_short_buffers_rejected_at_every_decode_position(G):
    import long_context_gsa_b200.workloads as W
    cfg = W.scaled(W.LLAMA_8X, batch=2, context=64 * 8)
    x = W.decode_inputs(cfg, device="cuda", own_len=3)
    B, hq, d = x["q"].shape
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, x["gist_k"].shape[2], x["raw_k"].shape[2], cfg.topk, False,
                       0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    args = dict(q=x["q"], gist_k=x["gist_k"], gist_v=x["gist_v"], raw_k=x["raw_k"], raw_v=x["raw_v"],
                n_gists=x["n_gists"], own_len=x["own_len"], out=out, sel_idx=sel)
    G.gsa_decode(desc, **args, ws=ws)  # the full-size buffers are accepted
    torch.cuda.synchronize()
    for name, t in args.items():
        bad = dict(args)
        bad[name] = t.reshape(-1)[:-1]
        with pytest.raises(ValueError, match="holds"):
            G.gsa_decode(desc, **bad, ws=ws)
    assert G.gsa_workspace_status(ws) == 0


def test_short_buffers_rejected_for_prefill(G):
    import long_context_gsa_b200.workloads as W
    cfg = W.scaled(W.PREFILL_32K, batch=1, hq=4, hkv=2, chunk=16, n_chunks=20, topk=4)
    x = W.prefill_inputs(cfg, device="cuda")
    B, hq, L, d = x["q_raw"].shape
    N = x["k_gist"].shape[2]
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, N, L, cfg.topk, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_PREFILL), dtype=torch.uint8, device="cuda")
    out_raw = torch.empty((B, hq, L, d), dtype=torch.float32, device="cuda")
    out_gist = torch.empty((B, hq, N, d), dtype=torch.float32, device="cuda")
    names = ("q_raw", "k_raw", "v_raw", "q_gist", "k_gist", "v_gist")
    for i in range(len(names) + 2):
        ins = [x[k] for k in names] + [out_raw, out_gist]
        ins[i] = ins[i].reshape(-1)[:-d]
        with pytest.raises(ValueError, match="holds"):
            G.gsa_prefill(desc, *ins, ws=ws)
