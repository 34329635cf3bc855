"""Causal GSA prefill on the GPU (tensor-core scoring + selection, tensor-core
gist attention, gathered raw tokens) against the float64 oracle, through the
C ABI.  Raw rows compare selections (tie window as in decode) and outputs;
gist rows compare outputs."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from _parity import TOL, tie_window

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


def run_gpu(x, cfg, exclude, split=False):
    B, hq, L, d = x["q_raw"].shape
    hkv, N = x["k_raw"].shape[1], x["k_gist"].shape[2]
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, N, L, cfg.topk, exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_PREFILL), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    out_raw = torch.full((B, hq, L, d), float("nan"), dtype=torch.float32, device="cuda")
    out_gist = torch.full((B, hq, N, d), float("nan"), dtype=torch.float32, device="cuda")
    sel = torch.full((B, hq, L, cfg.topk), -9, dtype=torch.int32, device="cuda")
    ssc = torch.empty((B, hq, L, cfg.topk), dtype=torch.float32, device="cuda")
    if split:
        G.gsa_prefill_score(desc, x["q_raw"], x["q_gist"], x["k_gist"], sel, ssc, ws)
        G.gsa_prefill_attend(desc, x["q_raw"], x["k_raw"], x["v_raw"], x["q_gist"], x["k_gist"], x["v_gist"], sel, ssc,
                             out_raw, out_gist, ws)
    else:
        G.gsa_prefill(desc, x["q_raw"], x["k_raw"], x["v_raw"], x["q_gist"], x["k_gist"], x["v_gist"], out_raw, out_gist,
                      sel, ssc, ws)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    return out_raw, out_gist, sel


def check(x, cfg, exclude, rows=None, what=""):
    """rows: oracle row ids ((b*hq+h)*(L+N) + pos); None = all rows."""
    out_raw, out_gist, sel = run_gpu(x, cfg, exclude)
    B, hq, L, d = x["q_raw"].shape
    hkv, N = x["k_raw"].shape[1], x["k_gist"].shape[2]
    P = L + N
    if rows is None:
        rows = np.arange(B * hq * P)
    rows = np.asarray(rows, dtype=np.int64)
    tk = W.to_oracle
    args = [tk(x[k]) for k in ("q_raw", "k_raw", "v_raw", "q_gist", "k_gist", "v_gist")]
    orc = oracle.get().prefill(*args, chunk=cfg.chunk, topk=cfg.topk, exclude=exclude, rows=rows)
    g_raw = out_raw.reshape(B * hq * L, d).cpu().numpy()
    g_gist = out_gist.reshape(B * hq * N, d).cpu().numpy()
    g_sel = sel.reshape(B * hq * L, cfg.topk).cpu().numpy()
    qr = W.to_oracle(x["q_raw"])
    kg = W.to_oracle(x["k_gist"])
    as64 = (lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)) if qr.dtype == np.uint16 else \
        (lambda a: a.astype(np.float64))
    scale = 1.0 / np.sqrt(d)
    G_ = hq // hkv
    worst, exempt, forced = 0.0, 0, []
    for i, r in enumerate(rows):
        bh, pos = divmod(int(r), P)
        b, h = divmod(bh, hq)
        if pos >= L:
            got = g_gist[bh * N + (pos - L)]
        else:
            got = g_raw[bh * L + pos]
            m = pos // cfg.chunk
            gs = set(int(t) for t in g_sel[bh * L + pos] if t >= 0)
            os = set(int(t) for t in orc["sel"][i] if t >= 0)
            if gs != os:
                s = scale * (as64(kg[b, h // G_, :m]) @ as64(qr[b, h, pos]))
                ex, lo, hi = tie_window(s, cfg.topk)
                assert ex and len(gs) == len(os) and all(lo <= s[t] <= hi for t in gs ^ os), \
                    f"{what}: selection differs outside the tie window at row {r} (pos {pos})"
                exempt += 1
                forced.append((i, r, sorted(gs) + [-1] * (cfg.topk - len(gs))))
                continue
        err = float(np.abs(got - orc["out"][i]).max())
        assert err <= TOL["bf16"], f"{what}: row {r} (pos {pos}, gist={pos >= L}) max abs err {err}"
        worst = max(worst, err)
    if forced:
        fr = oracle.get().prefill(*args, chunk=cfg.chunk, topk=cfg.topk, exclude=exclude,
                                  rows=np.array([f[1] for f in forced]), sel_in=np.array([f[2] for f in forced]))
        for j, (i, r, _) in enumerate(forced):
            bh, pos = divmod(int(r), P)
            err = float(np.abs(g_raw[bh * L + pos] - fr["out"][j]).max())
            assert err <= TOL["bf16"], f"{what}: tie-exempt row {r} max abs err {err}"
    return {"max_abs_err": worst, "tie_exempt": exempt, "rows": len(rows)}


SMALL = [
    ("n40_c16_k4", dict(batch=1, hq=4, hkv=2, chunk=16, n_chunks=40, topk=4)),
    ("n300_c8_k16", dict(batch=1, hq=8, hkv=2, chunk=8, n_chunks=300, topk=16)),
    ("ragged_tile_n37", dict(batch=2, hq=2, hkv=1, chunk=16, n_chunks=37, topk=5)),
    ("k16_n520_c4", dict(batch=1, hq=4, hkv=1, chunk=4, n_chunks=520, topk=16)),
    ("k1_n200_c8", dict(batch=1, hq=2, hkv=2, chunk=8, n_chunks=200, topk=1)),
    # d = 64 (the Llama-3.2-1B head size)
    ("d64_n300_c8_k16", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, n_chunks=300, topk=16)),
    ("d64_ragged_n37", dict(batch=2, hq=4, hkv=1, d=64, chunk=16, n_chunks=37, topk=5)),
    ("d64_k1_n150_c4", dict(batch=1, hq=4, hkv=4, d=64, chunk=4, n_chunks=150, topk=1)),
    # k > 16 (the wide scorer)
    ("k64_n300_c8_d64", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, n_chunks=300, topk=64)),
    ("k32_n200_c16_d128", dict(batch=1, hq=4, hkv=2, d=128, chunk=16, n_chunks=200, topk=32)),
    ("k17_ragged_n45_d64", dict(batch=2, hq=2, hkv=1, d=64, chunk=16, n_chunks=45, topk=17)),
    ("k64_n140_c4_d128", dict(batch=1, hq=4, hkv=1, d=128, chunk=4, n_chunks=140, topk=64)),
]


@pytest.mark.parametrize("name,chg", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("exclude", [False, True], ids=["default", "exclude"])
def test_small(name, chg, exclude):
    cfg = W.scaled(W.PREFILL_32K, seed=zlib.crc32(name.encode()), **chg)
    x = W.prefill_inputs(cfg, device="cuda")
    print(name, check(x, cfg, exclude, what=name))


def test_split_calls_match_fused():
    cfg = W.scaled(W.PREFILL_32K, batch=1, hq=4, hkv=2, chunk=16, n_chunks=100, topk=8)
    x = W.prefill_inputs(cfg, device="cuda")
    a = run_gpu(x, cfg, False, split=False)
    b = run_gpu(x, cfg, False, split=True)
    assert torch.equal(a[2], b[2]) and torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def check_heads(x, cfg, exclude, heads, what="", exact_ties=False):
    """Every row (all raw positions and all gist positions) of the listed
    (b, h) heads against the oracle, with vectorised set comparison; rows
    whose selections differ go through the tie rule.  With exact_ties, two
    chunks with bit-identical oracle scores on opposite sides of the
    boundary are a failure (the lower index must win), whatever the window."""
    out_raw, out_gist, sel = run_gpu(x, cfg, exclude)
    B, hq, L, d = x["q_raw"].shape
    hkv, N = x["k_raw"].shape[1], x["k_gist"].shape[2]
    P = L + N
    G_ = hq // hkv
    tk = W.to_oracle
    args = [tk(x[k]) for k in ("q_raw", "k_raw", "v_raw", "q_gist", "k_gist", "v_gist")]
    qr, kg = args[0], args[4]
    as64 = lambda a: (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # noqa: E731
    scale = 1.0 / np.sqrt(d)
    g_raw = out_raw.reshape(B * hq, L, d).cpu().numpy()
    g_gist = out_gist.reshape(B * hq, N, d).cpu().numpy()
    g_sel = np.sort(sel.reshape(B * hq, L, cfg.topk).cpu().numpy(), axis=-1)
    o = oracle.get()
    stats = {"rows": 0, "sel_rows": 0, "tie_exempt": 0, "exact_tie_rows": 0, "max_abs_err": 0.0}
    for bh in heads:
        b, h = divmod(bh, hq)
        orc = o.prefill(*args, chunk=cfg.chunk, topk=cfg.topk, exclude=exclude, rows=np.arange(bh * P, (bh + 1) * P))
        o_sel = np.sort(orc["sel"][:L], axis=-1)
        diff = np.nonzero((o_sel != g_sel[bh]).any(axis=1))[0]
        forced = []
        for pos in diff:
            m = pos // cfg.chunk
            gs = set(int(t) for t in g_sel[bh, pos] if t >= 0)
            os_ = set(int(t) for t in o_sel[pos] if t >= 0)
            s = scale * (as64(kg[b, h // G_, :m]) @ as64(qr[b, h, pos]))
            if exact_ties:
                lost = [s[t] for t in os_ - gs]
                assert not any(s[t] in lost for t in gs - os_), \
                    f"{what}: head {bh} pos {pos}: an exact tie went to the higher chunk index"
            ex, lo, hi = tie_window(s, cfg.topk)
            assert ex and len(gs) == len(os_) and all(lo <= s[t] <= hi for t in gs ^ os_), \
                f"{what}: head {bh} pos {pos}: selection differs outside the tie window"
            forced.append((pos, sorted(gs) + [-1] * (cfg.topk - len(gs))))
        stats["tie_exempt"] += len(forced)
        if exact_ties:
            stats["exact_tie_rows"] += int(sum(1 for pos in range(cfg.chunk * (cfg.topk + 1), L)
                                              if _boundary_tie(kg, qr, b, h // G_, h, pos, cfg, as64, scale)))
        keep = np.ones(L, bool)
        keep[[p_ for p_, _ in forced]] = False
        err_raw = np.abs(g_raw[bh][keep] - orc["out"][:L][keep]).max(initial=0.0)
        err_gist = np.abs(g_gist[bh] - orc["out"][L:]).max(initial=0.0)
        assert err_raw <= TOL["bf16"], f"{what}: head {bh} raw rows max abs err {err_raw}"
        assert err_gist <= TOL["bf16"], f"{what}: head {bh} gist rows max abs err {err_gist}"
        if forced:
            fr = o.prefill(*args, chunk=cfg.chunk, topk=cfg.topk, exclude=exclude,
                           rows=np.array([bh * P + p_ for p_, _ in forced]), sel_in=np.array([f for _, f in forced]))
            e = np.abs(g_raw[bh][[p_ for p_, _ in forced]] - fr["out"]).max()
            assert e <= TOL["bf16"], f"{what}: head {bh} tie-exempt rows max abs err {e}"
        stats["rows"] += P
        stats["sel_rows"] += L
        stats["max_abs_err"] = max(stats["max_abs_err"], float(err_raw), float(err_gist))
    return stats


def _boundary_tie(kg, qr, b, kvh, h, pos, cfg, as64, scale):
    """True when the oracle's k-th and (k+1)-th visible scores of this raw row are equal."""
    m = pos // cfg.chunk
    if m <= cfg.topk:
        return False
    s = np.sort(scale * (as64(kg[b, kvh, :m]) @ as64(qr[b, h, pos])))[::-1]
    return s[cfg.topk - 1] == s[cfg.topk]


def test_full_size_every_row():
    """The 32K-token prefill (28/4 heads, 2048 chunks of 16, top-16): every raw
    row's selection and output and every gist row's output, all 28 heads,
    against the oracle (974,848 rows)."""
    cfg = W.PREFILL_32K
    x = W.prefill_inputs(cfg, device="cuda")
    res = check_heads(x, cfg, False, range(cfg.batch * cfg.hq), what="prefill_32k")
    assert res["rows"] == cfg.hq * (cfg.length + cfg.n_chunks)
    print("prefill_32k default, every row:", res)


def test_full_size_every_row_exclude():
    """Exclude-unselected mode at full size: every row of four whole heads
    (one per kv head) against the oracle."""
    cfg = W.PREFILL_32K
    x = W.prefill_inputs(cfg, device="cuda")
    res = check_heads(x, cfg, True, (0, 9, 17, 27), what="prefill_32k exclude")
    print("prefill_32k exclude, 4 heads:", res)


def test_full_size_llama_heads():
    """The Llama-3.2-1B-shaped 32K prefill (32/8 heads, d = 64, 4096 chunks
    of 8, top-64): every row of four whole heads (two kv heads, first and
    last query head of each) against the oracle in default mode, and two
    heads in exclude mode."""
    cfg = W.PREFILL_LLAMA_32K
    x = W.prefill_inputs(cfg, device="cuda")
    res = check_heads(x, cfg, False, (0, 3, 28, 31), what="prefill_llama1b_32k")
    assert res["rows"] == 4 * (cfg.length + cfg.n_chunks)
    print("prefill_llama1b_32k default, 4 heads:", res)
    res = check_heads(x, cfg, True, (5, 18), what="prefill_llama1b_32k exclude")
    print("prefill_llama1b_32k exclude, 2 heads:", res)


@pytest.mark.parametrize("exclude", [False, True], ids=["default", "exclude"])
def test_exact_ties_through_prefill(exclude):
    """Gist keys repeated in runs of three (chunks 3j, 3j+1, 3j+2 share one
    key), so the k-th place of most rows falls inside a run of bit-equal
    scores: the selection must take the lower chunk indices ([nl] Selectie,
    ties to the lower index), under the causal limit of every row."""
    cfg = W.scaled(W.PREFILL_32K, seed=zlib.crc32(b"prefill_ties"), batch=1, hq=4, hkv=2, chunk=16, n_chunks=160,
                   topk=8)
    x = W.prefill_inputs(cfg, device="cuda")
    N = cfg.n_chunks
    src = torch.arange(N, device="cuda") // 3 * 3
    x["k_gist"] = x["k_gist"][:, :, src].contiguous()
    res = check_heads(x, cfg, exclude, range(cfg.batch * cfg.hq), what="prefill ties", exact_ties=True)
    assert res["exact_tie_rows"] > cfg.hq * 100, res  # the boundary really sits inside a run in most rows
    print("prefill exact ties:", res)


@pytest.mark.parametrize("topk", [8, 40], ids=["k8", "k40"])
def test_exact_ties_through_prefill_d64(topk):
    """The tie case of test_exact_ties_through_prefill at d = 64, with the
    narrow (k <= 16) and the wide scorer."""
    cfg = W.scaled(W.PREFILL_LLAMA_32K, seed=zlib.crc32(b"prefill_ties_d64"), batch=1, hq=4, hkv=2, chunk=8,
                   n_chunks=200, topk=topk)
    x = W.prefill_inputs(cfg, device="cuda")
    src = torch.arange(cfg.n_chunks, device="cuda") // 3 * 3
    x["k_gist"] = x["k_gist"][:, :, src].contiguous()
    res = check_heads(x, cfg, False, range(cfg.batch * cfg.hq), what="prefill ties d64", exact_ties=True)
    assert res["exact_tie_rows"] > cfg.hq * 100, res
    print("prefill exact ties d64:", res)
