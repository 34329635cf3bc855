"""Top-p (nucleus) chunk selection on the GPU (gsa_topp_select) against the
oracle's top-p step on the same fp32 scores.

The GPU sums the probabilities in fp32, the oracle in fp64, so the number
of chunks may differ by one only where the oracle's prefix mass lies within
MASS_TOL of top_p at the boundary (just below it before the last chosen
chunk, or just above it at that chunk).  Whatever the count, the chosen set
must be exactly the oracle's rank-order prefix of that length (ties to the
lower index), in ascending chunk order, with the scores as given.  A small
decode step then runs the unfold on a top-p selection (variable length,
-1 padded) against the oracle re-run with that selection."""
import zlib

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
MASS_TOL = 2e-5

G = None
W = None


@pytest.fixture(scope="module", autouse=True)
def _setup():
    global G, W
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G_
    import long_context_gsa_b200.workloads as W_
    G, W = G_, W_
    torch.cuda.init()


def _scores(rng, shape, dist):
    if dist == "randn3":  # a peaked softmax: a few chunks carry most of the mass
        return (3.0 * rng.standard_normal(shape)).astype(np.float32)
    if dist == "randn":
        return rng.standard_normal(shape).astype(np.float32)
    if dist == "ties8":
        return (rng.integers(-4, 4, size=shape) * 0.5).astype(np.float32)
    if dist == "flat":  # all equal: ceil(p * n) chunks, the lowest indices
        return np.zeros(shape, np.float32)
    raise ValueError(dist)


CASES = [
    # name, batch, hq, n_max, k, n_gists per batch
    ("llama_shape", 2, 32, 4096, 64, [4096, 3001]),
    ("qwen_shape", 1, 28, 8192, 128, [8192]),
    ("short_rows", 2, 8, 100, 64, [100, 40]),
    ("k_256", 1, 8, 2048, 256, [2048]),
    ("k_above_n", 2, 4, 48, 64, [48, 1]),
    ("empty_rows", 2, 4, 256, 16, [0, 256]),
    ("long_rows", 1, 4, 16384, 32, [16384]),
]


def _check(s, ng, hq, k, top_p, got, got_s, got_c):
    B = len(ng)
    n_valid = np.repeat(np.array(ng, np.int32), hq)
    flat = s.reshape(B * hq, -1).astype(np.float64)
    o = oracle.get().topp(flat, n_valid, k, top_p)
    for r in range(B * hq):
        c, oc = int(got_c[r]), int(o["count"][r])
        if c != oc:
            near = (c == oc - 1 and abs(top_p - o["mass_lo"][r]) <= MASS_TOL) or \
                   (c == oc + 1 and abs(o["mass_hi"][r] - top_p) <= MASS_TOL)
            assert near, (r, c, oc, o["mass_lo"][r], o["mass_hi"][r], top_p)
        want, want_s = oracle.get().topk(flat[r:r + 1], n_valid[r:r + 1], c)
        assert list(got[r][:c]) == list(want[0]), (r, got[r][:12], want[0][:12])
        np.testing.assert_array_equal(got_s[r][:c].astype(np.float64), want_s[0])
        assert (got[r][c:] == -1).all() and (got_s[r][c:] == -np.inf).all()


@pytest.mark.parametrize("top_p", [0.05, 0.5, 0.9, 0.999, 1.0])
@pytest.mark.parametrize("dist", ["randn3", "randn", "ties8", "flat"])
@pytest.mark.parametrize("name,B,hq,n_max,k,ng", CASES, ids=[c[0] for c in CASES])
def test_topp_matches_oracle(name, B, hq, n_max, k, ng, dist, top_p):
    if name in ("qwen_shape", "long_rows", "k_256") and top_p not in (0.5, 0.999):
        pytest.skip("large rows: two thresholds suffice")
    rng = np.random.default_rng(zlib.crc32(f"{name}/{dist}/{top_p}".encode()))
    s = _scores(rng, (B, hq, n_max), dist)
    for b in range(B):
        s[b, :, ng[b]:] = np.nan  # past the row's count: never read
    dev = torch.device("cuda")
    hkv = {32: 8, 28: 4, 8: 2, 4: 1}[hq]
    desc = G.make_desc(B, hq, hkv, 64, 8, n_max, n_max * 8, k, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    sel = torch.full((B, hq, k), -7, dtype=torch.int32, device=dev)
    ssc = torch.zeros((B, hq, k), dtype=torch.float32, device=dev)
    cnt = torch.full((B, hq), -7, dtype=torch.int32, device=dev)
    G.gsa_topp_select(desc, torch.from_numpy(s).to(dev), torch.tensor(ng, dtype=torch.int32, device=dev), top_p,
                      sel, ssc, cnt, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    got = sel.cpu().numpy().reshape(B * hq, k)
    got_s = ssc.cpu().numpy().reshape(B * hq, k)
    got_c = cnt.cpu().numpy().reshape(B * hq)
    _check(s, ng, hq, k, top_p, got, got_s, got_c)


@pytest.mark.parametrize("exclude", [False, True], ids=["default", "exclude"])
def test_topp_decode_step(exclude):
    """score -> top-p -> unfold on a small bf16 decode problem; the output
    is compared with the oracle run on the GPU's (variable-length) selection."""
    from _parity import TOL
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, context=300 * 8, topk=32)
    x = W.decode_inputs(cfg, device="cuda", seed=zlib.crc32(b"topp_decode"))
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, cfg.topk, exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    scores = torch.empty((B, hq, n_max), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device="cuda")
    cnt = torch.empty((B, hq), dtype=torch.int32, device="cuda")
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    G.gsa_score_gists(desc, x["q"], x["gist_k"], x["gist_v"], x["n_gists"], scores, ws)
    G.gsa_topp_select(desc, scores, x["n_gists"], 0.8, sel, ssc, cnt, ws)
    G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], sel, ssc,
                        G.GSA_PRIOR_NONE if exclude else G.GSA_PRIOR_GISTS, out, None, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    c = cnt.cpu().numpy().reshape(-1)
    assert (c >= 1).all() and (c <= cfg.topk).all()
    tk = W.to_oracle
    orc = oracle.get().decode(tk(x["q"]), tk(x["gist_k"]), tk(x["gist_v"]), tk(x["raw_k"]), tk(x["raw_v"]),
                              tk(x["n_gists"]), tk(x["own_len"]), chunk=cfg.chunk, topk=cfg.topk, exclude=exclude,
                              sel_in=sel.cpu().numpy().reshape(B * hq, cfg.topk))
    err = np.abs(out.cpu().numpy().reshape(B * hq, d) - orc["out"]).max()
    assert err <= TOL["bf16"], err


def test_topp_full_size_decode():
    """The full-size 32K-context, batch-16 decode with top-p (p = 0.1, at
    most 64 chunks): every row's selection against the oracle's top-p step
    on the GPU's scores, and every row's output against the oracle run with
    the GPU's selection."""
    from _parity import TOL
    cfg = W.LLAMA_8X
    x = W.decode_inputs(cfg, device="cuda")
    B, hq, d = x["q"].shape
    n_max, t_max = x["gist_k"].shape[2], x["raw_k"].shape[2]
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max, t_max, cfg.topk, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    scores = torch.empty((B, hq, n_max), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device="cuda")
    cnt = torch.empty((B, hq), dtype=torch.int32, device="cuda")
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    G.gsa_score_gists(desc, x["q"], x["gist_k"], x["gist_v"], x["n_gists"], scores, ws)
    G.gsa_topp_select(desc, scores, x["n_gists"], 0.1, sel, ssc, cnt, ws)
    G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], sel, ssc,
                        G.GSA_PRIOR_GISTS, out, None, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    ng = x["n_gists"].cpu().tolist()
    _check(scores.cpu().numpy(), ng, hq, cfg.topk, 0.1, sel.cpu().numpy().reshape(B * hq, -1),
           ssc.cpu().numpy().reshape(B * hq, -1), cnt.cpu().numpy().reshape(-1))
    tk = W.to_oracle
    orc = oracle.get().decode(tk(x["q"]), tk(x["gist_k"]), tk(x["gist_v"]), tk(x["raw_k"]), tk(x["raw_v"]),
                              tk(x["n_gists"]), tk(x["own_len"]), chunk=cfg.chunk, topk=cfg.topk,
                              sel_in=sel.cpu().numpy().reshape(B * hq, cfg.topk))
    err = np.abs(out.cpu().numpy().reshape(B * hq, d) - orc["out"]).max()
    assert err <= TOL["bf16"], err
    print("llama1b_8x top-p decode: max abs err", err, "chunks mean", float(cnt.float().mean()))
