"""The gist-position step at chunk completion (gsa_gist_step) on the GPU
against the float64 oracle, through the C ABI: the new gist is written at
gist row N (bit-exact), the gist query's attention over gists 0..N and the
own chunk's raw rows matches the oracle within the output tolerance, and the
counts advance (n_gists = N + 1, own_len = 0).  A sequence with a full gist
array is flagged and attends the completed gists and its raw rows only."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from _parity import TOL

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


def run_gpu(x, cfg, out_bf16=False):
    B, hq, d = x["q"].shape
    hkv, n_max, t_max = x["gist_k"].shape[1], x["gist_k"].shape[2], x["raw_k"].shape[2]
    dt = G.GSA_BF16 if x["q"].dtype == torch.bfloat16 else G.GSA_F32
    desc = G.make_desc(B, hq, hkv, d, cfg.chunk, n_max, t_max, cfg.topk, cfg.exclude, 0.0, dt,
                       G.GSA_BF16 if out_bf16 else G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_GIST_STEP), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    st = {k: x[k].clone() for k in ("gist_k", "gist_v", "n_gists", "own_len")}
    out = torch.empty((B, hq, d), dtype=torch.bfloat16 if out_bf16 else torch.float32, device="cuda")
    lse = torch.empty((B, hq), dtype=torch.float32, device="cuda")
    G.gsa_gist_step(desc, x["q"], x["k_new"], x["v_new"], st["gist_k"], st["gist_v"], x["raw_k"], x["raw_v"],
                    st["n_gists"], st["own_len"], out, lse, ws)
    torch.cuda.synchronize()
    return out, lse, st, G.gsa_workspace_status(ws)


def run_oracle(x, cfg):
    tk = W.to_oracle
    return oracle.get().gist_step(tk(x["q"]), tk(x["k_new"]), tk(x["v_new"]), tk(x["gist_k"]), tk(x["gist_v"]),
                                  tk(x["raw_k"]), tk(x["raw_v"]), tk(x["n_gists"]), tk(x["own_len"]), chunk=cfg.chunk)


def check(x, cfg, what, out_bf16=False):
    out, lse, st, flags = run_gpu(x, cfg, out_bf16)
    assert flags == 0, f"{what}: device status {flags:#x}"
    B, hq, d = x["q"].shape
    n0 = x["n_gists"].cpu().numpy()
    # bookkeeping: exact
    assert st["n_gists"].cpu().tolist() == (n0 + 1).tolist()
    assert st["own_len"].cpu().tolist() == [0] * B
    for b in range(B):
        N = int(n0[b])
        assert torch.equal(st["gist_k"][b, :, N], x["k_new"][b]) and torch.equal(st["gist_v"][b, :, N], x["v_new"][b])
        keep = [m for m in range(x["gist_k"].shape[2]) if m != N]
        assert torch.equal(st["gist_k"][b, :, keep], x["gist_k"][b, :, keep])
        assert torch.equal(st["gist_v"][b, :, keep], x["gist_v"][b, :, keep])
    ref = run_oracle(x, cfg)
    dtype = "bf16" if x["q"].dtype == torch.bfloat16 else "f32"
    got = out.float().cpu().numpy().reshape(B * hq, d)
    tol = TOL[dtype] + (np.abs(ref["out"]).max() * 2.0 ** -8 if out_bf16 else 0.0)
    err = np.abs(got - ref["out"]).max()
    assert err <= tol, f"{what}: max abs err {err}"
    lerr = np.abs(lse.cpu().numpy().reshape(-1) - ref["lse"]).max()
    assert lerr <= 1e-4 * max(1.0, np.abs(ref["lse"]).max()), f"{what}: lse err {lerr}"
    return err


CASES = [
    # name, config changes, ragged gist counts
    ("gqa4_d64", dict(batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 300), [300, 123]),
    ("gqa4_d128_c16", dict(batch=2, hq=8, hkv=2, d=128, chunk=16, context=16 * 200), [200, 1]),
    ("first_chunk", dict(batch=2, hq=4, hkv=1, d=64, chunk=8, context=8 * 40), [0, 40]),
    ("gqa7_d128", dict(batch=1, hq=28, hkv=4, d=128, chunk=16, context=16 * 513), None),
    ("mha_long", dict(batch=1, hq=4, hkv=4, d=64, chunk=4, context=4 * 5000), None),
]


@pytest.mark.parametrize("name,chg,ragged", CASES, ids=[c[0] for c in CASES])
def test_small_bf16(name, chg, ragged):
    cfg = W.scaled(W.LLAMA_8X, **chg)
    x = W.gist_step_inputs(cfg, device="cuda", seed=zlib.crc32(name.encode()), ragged=ragged)
    check(x, cfg, name)


def test_f32_and_bf16_out():
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 77, dtype="f32")
    x = W.gist_step_inputs(cfg, device="cuda", seed=3, ragged=[77, 10])
    check(x, cfg, "f32")
    cfg2 = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=128, chunk=8, context=8 * 77)
    check(W.gist_step_inputs(cfg2, device="cuda", seed=4), cfg2, "bf16 out", out_bf16=True)


def test_partial_own_chunk():
    """own_len < chunk is allowed: the gist query sees the raw rows present."""
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 64)
    x = W.gist_step_inputs(cfg, device="cuda", seed=9, own_len=3)
    check(x, cfg, "own 3")


def test_full_gist_array_is_flagged():
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 64)
    x = W.gist_step_inputs(cfg, device="cuda", seed=11)
    n_max = x["gist_k"].shape[2]
    x["n_gists"] = torch.tensor([n_max, 20], dtype=torch.int32, device="cuda")
    out, lse, st, flags = run_gpu(x, cfg)
    assert flags & G.GSA_DEVERR_CAPACITY
    assert st["n_gists"].cpu().tolist() == [n_max, 21] and st["own_len"].cpu().tolist() == [8, 0]
    assert torch.equal(st["gist_k"][0], x["gist_k"][0])
    # batch 0: gists 0..n_max-1 and the raw rows at n_max*chunk (the decode's compression-only set)
    tk = W.to_oracle
    t_need = (n_max + 1) * cfg.chunk
    raw_k = torch.cat([x["raw_k"], torch.zeros_like(x["raw_k"][:, :, :cfg.chunk])], 2)[:, :, :t_need]
    raw_v = torch.cat([x["raw_v"], torch.zeros_like(x["raw_v"][:, :, :cfg.chunk])], 2)[:, :, :t_need]
    ref = oracle.get().decode(tk(x["q"][:1]), tk(x["gist_k"][:1]), tk(x["gist_v"][:1]), tk(raw_k[:1]),
                              tk(raw_v[:1]), np.array([n_max], np.int32), np.array([0], np.int32), chunk=cfg.chunk,
                              topk=0)
    got = out[0].cpu().numpy().reshape(-1, x["q"].shape[2])
    assert np.abs(got - ref["out"]).max() <= TOL["bf16"]


def test_chunk_completion_loop():
    """Three chunk completions in a row on the same arrays: each step's gist
    becomes a completed gist of the next (as a decode loop would do)."""
    cfg = W.scaled(W.LLAMA_8X, batch=2, hq=8, hkv=2, d=64, chunk=8, context=8 * 50)
    x = W.gist_step_inputs(cfg, device="cuda", seed=21, ragged=[40, 7])
    n_max = x["gist_k"].shape[2]
    x["gist_k"] = torch.cat([x["gist_k"], torch.zeros_like(x["gist_k"][:, :, :3])], 2)
    x["gist_v"] = torch.cat([x["gist_v"], torch.zeros_like(x["gist_v"][:, :, :3])], 2)
    gen = torch.Generator(device="cuda").manual_seed(5)
    B, hq, d = x["q"].shape
    dev = "cuda"
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, n_max + 3, x["raw_k"].shape[2], 0, False, 0.0, G.GSA_BF16,
                       G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_GIST_STEP), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    for step in range(3):
        snap = {k: x[k].clone() for k in ("gist_k", "gist_v", "n_gists")}
        q = torch.randn((B, hq, d), generator=gen, device=dev).to(torch.bfloat16)
        kn = torch.randn((B, cfg.hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        vn = torch.randn((B, cfg.hkv, d), generator=gen, device=dev).to(torch.bfloat16)
        own = torch.full((B,), cfg.chunk, dtype=torch.int32, device=dev)
        out = torch.empty((B, hq, d), dtype=torch.float32, device=dev)
        G.gsa_gist_step(desc, q, kn, vn, x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], own, out,
                        None, ws)
        torch.cuda.synchronize()
        assert G.gsa_workspace_status(ws) == 0
        tk = W.to_oracle
        ref = oracle.get().gist_step(tk(q), tk(kn), tk(vn), tk(snap["gist_k"]), tk(snap["gist_v"]), tk(x["raw_k"]),
                                     tk(x["raw_v"]), tk(snap["n_gists"]), np.full(B, cfg.chunk, np.int32),
                                     chunk=cfg.chunk)
        assert own.cpu().tolist() == [0] * B  # the step zeroed the own counts
        assert np.abs(out.cpu().numpy().reshape(B * hq, d) - ref["out"]).max() <= TOL["bf16"]
        assert x["n_gists"].cpu().tolist() == [41 + step, 8 + step]


@pytest.mark.parametrize("name", ["llama1b_8x", "qwen7b_16x"])
def test_full_size(name):
    """Chunk completion for every sequence of the full-size decode workloads
    (32K context, batch 16, GQA 4; 128K context, batch 4, GQA 7); every row
    is compared."""
    cfg = W.CONFIGS[name]
    x = W.gist_step_inputs(cfg, device="cuda")
    err = check(x, cfg, name + " gist step")
    print(name, "gist step max abs err", err)
