"""Backward of a decode step for a fixed selection (gsa_decode_backward) on
the GPU against the float64 oracle, through the C ABI.

The GPU forward runs first (gsa_decode) and gives the selection, the output
and the log-sum-exp; the backward takes those and a random fp32 d_out.  The
oracle is run with the GPU's selection (selection parity is covered by the
forward tests), so every gradient element is compared.  Both sides read the
same bf16 / fp32 inputs; the GPU works in fp32 and adds each key / value row
from every head of its GQA group with atomics, so the bound is the
accumulation error of fp32 sums of a few thousand terms, relative to the
gradient's own scale: max|gpu - oracle| <= GRAD_RTOL * max(1, max|oracle|)."""
import zlib

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
GRAD_RTOL = {"bf16": 2e-4, "f32": 2e-5}
KEYS = ("d_q", "d_gist_k", "d_gist_v", "d_raw_k", "d_raw_v")

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


def run_gpu(x, cfg, exclude, d_out):
    dev = x["q"].device
    B, hq, d = x["q"].shape
    hkv, n_max, t_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2]
    dt = G.GSA_BF16 if x["q"].dtype == torch.bfloat16 else G.GSA_F32
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, exclude, 0.0, dt, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
    lse = torch.empty((B, hq), dtype=torch.float32, device=dev)
    k = max(cfg.topk, 1)
    sel = torch.full((B, hq, k), -7, dtype=torch.int32, device=dev)
    ssc = torch.empty((B, hq, k), dtype=torch.float32, device=dev)
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"], out, lse,
                 sel if cfg.topk else None, ssc if cfg.topk else None, ws)
    grads = {"d_q": torch.zeros((B, hq, d), dtype=torch.float32, device=dev)}
    for nm, src in (("d_gist_k", "gist_k"), ("d_gist_v", "gist_v"), ("d_raw_k", "raw_k"), ("d_raw_v", "raw_v")):
        grads[nm] = torch.zeros(x[src].shape, dtype=torch.float32, device=dev)
    G.gsa_decode_backward(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                          sel if cfg.topk else None, out, lse, d_out, grads["d_q"], grads["d_gist_k"],
                          grads["d_gist_v"], grads["d_raw_k"], grads["d_raw_v"])
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    return {k_: v.cpu().numpy() for k_, v in grads.items()}, sel.cpu().numpy()


def run_oracle(x, cfg, exclude, sel, d_out, batches=None):
    tk = W.to_oracle
    xs = x if batches is None else {k_: (v[batches] if torch.is_tensor(v) and v.dim() > 0 else v)
                                    for k_, v in x.items()}
    s = sel if batches is None else sel[batches]
    g = d_out if batches is None else d_out[batches]
    B, hq = xs["q"].shape[:2]
    return oracle.get().decode_backward(
        tk(xs["q"]), tk(xs["gist_k"]), tk(xs["gist_v"]), tk(xs["raw_k"]), tk(xs["raw_v"]), tk(xs["n_gists"]),
        tk(xs["own_len"]), s.reshape(B * hq, -1)[:, :cfg.topk] if cfg.topk else None, g.cpu().numpy(),
        chunk=cfg.chunk, topk=cfg.topk, exclude=exclude)


def compare(got, ref, dtype, what, batches=None):
    worst = {}
    for k_ in KEYS:
        g = got[k_] if batches is None else got[k_][batches]
        r = ref[k_]
        scale = max(1.0, float(np.abs(r).max()))
        err = float(np.abs(g - r).max())
        assert err <= GRAD_RTOL[dtype] * scale, f"{what}: {k_} max abs err {err} (scale {scale})"
        worst[k_] = err / scale
    return worst


def d_out_for(x, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.randn(x["q"].shape, generator=gen, dtype=torch.float32).to(x["q"].device)


SMALL = [
    # name, config changes, ragged gist counts, own_len
    ("gqa4_d128", dict(batch=2, hq=8, hkv=2, d=128, chunk=8, context=8 * 300, topk=16), [300, 141], 3),
    ("gqa4_d64_c16", dict(batch=1, hq=8, hkv=2, d=64, chunk=16, context=16 * 200, topk=32), None, 16),
    ("mha", dict(batch=2, hq=4, hkv=4, d=64, chunk=8, context=8 * 90, topk=8), [90, 5], 1),
    ("k_above_n", dict(batch=2, hq=4, hkv=1, d=128, chunk=8, context=8 * 40, topk=64), [40, 7], 2),
    ("no_gists", dict(batch=2, hq=4, hkv=2, d=64, chunk=8, context=8 * 30, topk=8), [0, 30], 4),
    ("topk0", dict(batch=1, hq=8, hkv=2, d=64, chunk=8, context=8 * 50, topk=0), None, 2),
    # a 16-head group with 200 selections each: many heads adding into the same rows
    ("g16_k200", dict(batch=1, hq=32, hkv=2, d=64, chunk=4, context=4 * 400, topk=200), [400], 2),
    # heads of a group choosing overlapping chunks (few gists, many heads)
    ("overlap_g7", dict(batch=1, hq=28, hkv=4, d=128, chunk=16, context=16 * 40, topk=16), None, 5),
]


@pytest.mark.parametrize("name,chg,ragged,own", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("exclude", [False, True], ids=["default", "exclude"])
def test_small_bf16(name, chg, ragged, own, exclude):
    if exclude and chg["topk"] == 0:
        pytest.skip("exclude with no selection attends only the own rows: covered by the topk0 default case")
    cfg = W.scaled(W.LLAMA_8X, **chg)
    x = W.decode_inputs(cfg, device="cuda", own_len=own, ragged=ragged, seed=zlib.crc32(name.encode()))
    d_out = d_out_for(x, zlib.crc32(name.encode()) + 1)
    got, sel = run_gpu(x, cfg, exclude, d_out)
    ref = run_oracle(x, cfg, exclude, sel, d_out)
    compare(got, ref, "bf16", name)


def test_small_f32():
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 120, topk=12, dtype="f32")
    x = W.decode_inputs(cfg, device="cuda", own_len=5, ragged=[120, 77], seed=77)
    d_out = d_out_for(x, 78)
    for excl in (False, True):
        got, sel = run_gpu(x, cfg, excl, d_out)
        compare(got, run_oracle(x, cfg, excl, sel, d_out), "f32", f"f32 exclude={excl}")


def test_accumulates():
    """The gradients are added to what the buffers hold: two calls give twice one call."""
    cfg = W.scaled(W.LLAMA_8X, batch=1, hq=8, hkv=2, d=64, chunk=8, context=8 * 64, topk=8, dtype="f32")
    x = W.decode_inputs(cfg, device="cuda", own_len=3, seed=5)
    d_out = d_out_for(x, 6)
    B, hq, d = x["q"].shape
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, x["gist_k"].shape[2], x["raw_k"].shape[2], cfg.topk, False, 0.0,
                       G.GSA_F32, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    out = torch.empty((B, hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, hq), dtype=torch.float32, device="cuda")
    sel = torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda")
    ssc = torch.empty((B, hq, cfg.topk), dtype=torch.float32, device="cuda")
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"], out, lse,
                 sel, ssc, ws)
    bufs = [torch.zeros((B, hq, d), device="cuda")] + [torch.zeros(x[s].shape, device="cuda")
                                                       for s in ("gist_k", "gist_v", "raw_k", "raw_v")]
    once = None
    for call in range(2):
        G.gsa_decode_backward(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"],
                              x["own_len"], sel, out, lse, d_out, *bufs)
        torch.cuda.synchronize()
        if call == 0:
            once = [b.clone() for b in bufs]
    for a, b in zip(once, bufs):
        torch.testing.assert_close(b, 2 * a, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("excl", [False, True], ids=["default", "exclude"])
def test_full_size_sampled_batches(excl):
    """The 32K-context, batch-16 workload on the GPU; the oracle recomputes
    the gradients of two whole batches (batch b's gradients depend on batch
    b's rows only), every element of which is compared."""
    cfg = W.LLAMA_8X
    x = W.decode_inputs(cfg, device="cuda")
    d_out = d_out_for(x, 99)
    got, sel = run_gpu(x, cfg, excl, d_out)
    for bsel in ([0], [cfg.batch - 1]):
        ref = run_oracle(x, cfg, excl, sel, d_out, batches=bsel)
        res = compare(got, ref, "bf16", f"llama1b_8x batch {bsel}", batches=bsel)
    print("llama1b_8x backward", "exclude" if excl else "default", res)


def test_full_size_qwen_one_batch():
    """The 128K-context Qwen-shaped workload (7 query heads per kv head, d = 128,
    top-128 of 8192 chunks of 16) on the GPU; the oracle recomputes batch 0's
    gradients, every element of which is compared."""
    cfg = W.QWEN_16X
    x = W.decode_inputs(cfg, device="cuda")
    d_out = d_out_for(x, 123)
    got, sel = run_gpu(x, cfg, False, d_out)
    ref = run_oracle(x, cfg, False, sel, d_out, batches=[0])
    res = compare(got, ref, "bf16", "qwen7b_16x batch 0", batches=[0])
    print("qwen7b_16x backward", res)
