"""Flat GSA decode on the GPU (score -> select -> unfold) against the float64
oracle, through the C ABI.  Needs a B200 and the built libgsa.so."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from _parity import check_rows

pytestmark = pytest.mark.gpu

W = None
G = None


@pytest.fixture(scope="module", autouse=True)
def _setup():
    global W, G
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G_
    import long_context_gsa_b200.workloads as W_
    W, G = W_, G_
    torch.cuda.init()


def run_gpu(x, cfg, exclude=None, out_bf16=False, fused=True):
    dev = x["q"].device
    B, hq, d = x["q"].shape
    hkv, n_max, t_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2]
    dt = G.GSA_BF16 if x["q"].dtype == torch.bfloat16 else G.GSA_F32
    excl = cfg.exclude if exclude is None else exclude
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, excl, 0.0, dt,
                       G.GSA_BF16 if out_bf16 else G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.bfloat16 if out_bf16 else torch.float32, device=dev)
    lse = torch.empty((B, hq), dtype=torch.float32, device=dev)
    k = max(cfg.topk, 1)
    sel = torch.full((B, hq, k), -7, dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, k), dtype=torch.float32, device=dev)
    scores = None
    if fused:
        G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                     out, lse, sel if cfg.topk else None, ssc if cfg.topk else None, ws)
    else:
        scores = torch.full((B, hq, n_max), float("nan"), dtype=torch.float32, device=dev)
        G.gsa_score_gists(desc, x["q"], x["gist_k"], None if excl else x["gist_v"], x["n_gists"], scores, ws)
        if cfg.topk:
            G.gsa_topk_select(desc, scores, x["n_gists"], sel, ssc, ws)
        G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"],
                            sel if cfg.topk else None, ssc if cfg.topk else None,
                            G.GSA_PRIOR_NONE if excl else G.GSA_PRIOR_GISTS, out, lse, ws)
    torch.cuda.synchronize()
    flags = G.gsa_workspace_status(ws)
    assert flags == 0, f"device status flags {flags:#x}"
    return out, lse, (sel if cfg.topk else torch.full((B, hq, 0), -1, dtype=torch.int32)), ssc, scores


def run_oracle(x, cfg, exclude=None, rows=None, sel_in=None):
    o = oracle.get()
    tk = W.to_oracle
    excl = cfg.exclude if exclude is None else exclude
    return o.decode(tk(x["q"]), tk(x["gist_k"]), tk(x["gist_v"]), tk(x["raw_k"]), tk(x["raw_v"]), tk(x["n_gists"]),
                    tk(x["own_len"]), chunk=cfg.chunk, topk=cfg.topk, exclude=excl, rows=rows, sel_in=sel_in,
                    want_scores=True)


def compare(x, cfg, exclude=None, out_bf16=False, rows=None, fused=True, what=""):
    out, lse, sel, ssc, scores = run_gpu(x, cfg, exclude, out_bf16, fused)
    B, hq, d = x["q"].shape
    all_rows = np.arange(B * hq) if rows is None else np.asarray(rows)
    orc = run_oracle(x, cfg, exclude, rows=all_rows)
    g_out = out.float().reshape(B * hq, d).cpu().numpy()[all_rows]
    g_sel = sel.reshape(B * hq, -1).cpu().numpy()[all_rows]

    def rerun(slots, forced):
        return run_oracle(x, cfg, exclude, rows=all_rows[slots], sel_in=forced)

    dtype = "bf16" if x["q"].dtype == torch.bfloat16 else "f32"
    res = check_rows(g_out, g_sel, orc, orc["scores"], cfg.topk, dtype, out_bf16, rerun, what)
    g_lse = lse.reshape(-1).cpu().numpy()[all_rows]
    ok = np.isfinite(orc["lse"])
    assert np.allclose(g_lse[ok], orc["lse"][ok], atol=1e-3 if dtype == "bf16" else 1e-5)
    if scores is not None:
        sc = scores.reshape(B * hq, -1).cpu().numpy()[all_rows]
        valid = ~np.isnan(orc["scores"])
        assert np.nanmax(np.abs(sc[valid] - orc["scores"][valid])) < (1e-3 if dtype == "bf16" else 1e-5)
    return res, g_sel


SMALL = [
    # name, cfg changes, n_max extra, ragged counts, own_len
    ("g7_d128_c16", dict(batch=2, hq=28, hkv=4, d=128, chunk=16, context=1000 * 16, topk=32), [1000, 617], 16),
    ("g4_d64_c8", dict(batch=2, hq=32, hkv=8, d=64, chunk=8, context=700 * 8, topk=64), [700, 700], 1),
    ("g16_d128", dict(batch=1, hq=16, hkv=1, d=128, chunk=16, context=333 * 16, topk=16), None, 5),
    ("g1_d64", dict(batch=2, hq=4, hkv=4, d=64, chunk=8, context=200 * 8, topk=8), [200, 150], 3),
    ("n_below_k", dict(batch=1, hq=8, hkv=2, d=128, chunk=16, context=20 * 16, topk=64), None, 7),
    ("k0", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, context=50 * 8, topk=0), None, 2),
    ("c32_full_own", dict(batch=1, hq=8, hkv=2, d=128, chunk=32, context=300 * 32, topk=24), None, 32),
    ("n0", dict(batch=2, hq=4, hkv=2, d=64, chunk=8, context=40 * 8, topk=4), [0, 40], 2),
    ("big_k", dict(batch=1, hq=4, hkv=1, d=64, chunk=4, context=3000 * 4, topk=700), None, 2),
    # one scoring CTA per (b, kv head): its thread groups select several rows each in turn
    ("one_split_many_rows_d64", dict(batch=2, hq=16, hkv=2, d=64, chunk=8, context=60 * 8, topk=8), [60, 41], 3),
    ("one_split_many_rows_d128", dict(batch=2, hq=28, hkv=4, d=128, chunk=16, context=60 * 16, topk=8), [60, 33], 5),
]


@pytest.mark.parametrize("name,chg,ragged,own", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("exclude", [False, True], ids=["default", "exclude"])
def test_small_bf16(name, chg, ragged, own, exclude):
    cfg = W.scaled(W.QWEN_16X, kv_std=1.0, **chg)
    x = W.decode_inputs(cfg, device="cuda", own_len=own, ragged=ragged, seed=zlib.crc32(name.encode()) % 100000)
    compare(x, cfg, exclude=exclude, what=name)


@pytest.mark.parametrize("d", [64, 128])
def test_small_f32(d):
    cfg = W.scaled(W.PR1, batch=2, hq=4, hkv=2, d=d, chunk=16, context=300 * 16, topk=12, dtype="f32")
    x = W.decode_inputs(cfg, device="cuda", own_len=9, ragged=[300, 211])
    compare(x, cfg, exclude=False, what=f"f32 d={d}")
    compare(x, cfg, exclude=True, what=f"f32 d={d} exclude")


def test_bf16_output():
    cfg = W.scaled(W.LLAMA_8X, batch=2, context=512 * 8)
    x = W.decode_inputs(cfg, device="cuda", own_len=4)
    compare(x, cfg, out_bf16=True, what="bf16 out")


def test_separate_entry_points_match_fused():
    """gsa_decode (selection in the unfold prologue) against the three
    separate calls (gsa_topk_select's own kernel): the same selection, and
    outputs equal up to fp32 summation order (the two launches may cut a
    row's unfold into different splits)."""
    cfg = W.scaled(W.QWEN_16X, batch=2, context=900 * 16, kv_std=1.0)
    x = W.decode_inputs(cfg, device="cuda", own_len=6)
    for excl in (False, True):
        a = run_gpu(x, cfg, excl, fused=True)
        b = run_gpu(x, cfg, excl, fused=False)
        assert torch.equal(a[2], b[2])
        assert torch.equal(a[3], b[3])  # selected scores
        assert (a[0] - b[0]).abs().max().item() <= 1e-5
    compare(x, cfg, fused=False, what="separate calls")


@pytest.mark.parametrize("excl", [False, True], ids=["default", "exclude"])
def test_score_select_entry_point(excl):
    """gsa_score_select (scoring with the selection in its tail) then
    gsa_unfold_attend computes the fused step, and its scores are
    gsa_score_gists's."""
    cfg = W.scaled(W.LLAMA_8X, batch=3, context=1500 * 8)
    x = W.decode_inputs(cfg, device="cuda", own_len=5, ragged=[1500, 999, 64])
    B, hq, d = x["q"].shape
    hkv, n_max, t_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2]
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, excl, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    scores = torch.full((B, hq, n_max), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, hq), dtype=torch.float32, device="cuda")
    sel = torch.full((B, hq, cfg.topk), -7, dtype=torch.int32, device="cuda")
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device="cuda")
    G.gsa_score_select(desc, x["q"], x["gist_k"], None if excl else x["gist_v"], x["n_gists"], scores, sel, ssc, ws)
    G.gsa_unfold_attend(desc, x["q"], x["raw_k"], x["raw_v"], x["gist_v"], x["n_gists"], x["own_len"], sel, ssc,
                        G.GSA_PRIOR_NONE if excl else G.GSA_PRIOR_GISTS, out, lse, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    a = run_gpu(x, cfg, excl, fused=True)
    b = run_gpu(x, cfg, excl, fused=False)
    assert torch.equal(a[2], sel) and torch.equal(a[3], ssc)
    assert (a[0] - out).abs().max().item() <= 1e-5 and (a[1] - lse).abs().max().item() <= 1e-5
    valid = torch.isfinite(b[4])
    assert torch.equal(scores[valid], b[4][valid])


TIE_CASES = [
    # gist keys repeated in runs of three: most rows' k-th place falls inside a run of equal scores
    ("runs_of_3", dict(batch=2, hq=32, hkv=8, d=64, chunk=8, context=2000 * 8, topk=64), 3),
    ("runs_of_3_d128", dict(batch=1, hq=28, hkv=4, d=128, chunk=16, context=3000 * 16, topk=128), 3),
    # every gist key equal: all scores of a row tie (the exact radix fallback)
    ("all_equal", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, context=3000 * 8, topk=64), 0),
    # fewer groups of 16 than k: the scores themselves are the bound's values
    ("few_groups", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, context=300 * 8, topk=64), 3),
    # a row longer than the group list (more than 16384 gists): the radix path
    ("long_row", dict(batch=1, hq=4, hkv=1, d=64, chunk=8, context=20000 * 8, topk=32), 3),
]


@pytest.mark.parametrize("name,chg,run", TIE_CASES, ids=[c[0] for c in TIE_CASES])
def test_exact_ties_go_to_lower_index(name, chg, run):
    """Bit-equal scores on both sides of the k-th place: the selection takes
    the lower chunk indices ([nl] Selectie; ties to the lower index), in the
    fused step as in gsa_topk_select, and matches the oracle."""
    cfg = W.scaled(W.QWEN_16X, kv_std=1.0, **chg)
    x = W.decode_inputs(cfg, device="cuda", own_len=3, seed=zlib.crc32(name.encode()) % 100000)
    N = cfg.n_gists
    src = torch.arange(N, device="cuda")
    src = src // run * run if run else torch.zeros_like(src)
    x["gist_k"] = x["gist_k"][:, :, src].contiguous()
    a = run_gpu(x, cfg, False, fused=True)
    b = run_gpu(x, cfg, False, fused=False)
    assert torch.equal(a[2], b[2]), f"{name}: fused and separate selections differ"
    B, hq, d = x["q"].shape
    rows = np.arange(B * hq)
    orc = run_oracle(x, cfg, rows=rows)
    g_sel = np.sort(a[2].reshape(B * hq, -1).cpu().numpy(), -1)
    o_sel = np.sort(orc["sel"], -1)
    exact_tie_rows = 0
    for r in rows:
        s = orc["scores"][r]
        srt = np.sort(s[~np.isnan(s)])[::-1]
        if len(srt) > cfg.topk and srt[cfg.topk - 1] == srt[cfg.topk]:
            exact_tie_rows += 1
        if not np.array_equal(g_sel[r], o_sel[r]):
            gs, os_ = set(g_sel[r].tolist()) - {-1}, set(o_sel[r].tolist()) - {-1}
            lost = {s[t] for t in os_ - gs}
            assert not any(s[t] in lost for t in gs - os_), f"{name}: row {r}: exact tie went to a higher index"
    assert exact_tie_rows > len(rows) // 2, (name, exact_tie_rows)
    compare(x, cfg, what=name)


def test_pr1_all_steps():
    """The tiny fp32 single-head workload: every one of its 64 decode steps."""
    static, steps = W.pr1_steps(device="cuda")
    cfg = W.PR1
    hits = 0
    for s, st in enumerate(steps):
        x = dict(static, q=st["q"], n_gists=st["n_gists"], own_len=st["own_len"])
        _, sel = compare(x, cfg, what=f"pr1 step {s}")
        hits += len(set(sel[0].tolist()) & set(static["planted"].tolist()))
    assert hits / (8 * len(steps)) > 0.9


@pytest.mark.parametrize("name", ["llama1b_8x", "llama1b_8x_excl", "qwen7b_16x", "qwen7b_16x_excl"])
def test_full_size(name):
    """Full-size workloads; every row is checked (the oracle needs seconds here)."""
    excl = name.endswith("_excl")
    cfg = W.CONFIGS[name[:-len("_excl")] if name == "llama1b_8x_excl" else name]
    x = W.decode_inputs(cfg, device="cuda")
    res, sel = compare(x, cfg, exclude=True if excl else None, what=name)
    planted = x["planted"].reshape(-1).numpy()
    recall = np.mean([planted[r] in set(sel[r].tolist()) for r in range(len(planted))])
    assert recall > 0.9, recall
    print(name, res, "planted recall", recall)
