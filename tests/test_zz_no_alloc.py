"""gsa_decode_noalloc: the decode step for callers that cannot allocate
device memory (a plugin or FFI host that only passes input/output pointers,
or a latency-critical caller that must not call cudaMalloc).  It uses the
library's built-in scratch array instead of a caller workspace, so its
results must equal gsa_decode's with a caller-allocated workspace, and the
device status it leaves is read with gsa_noalloc_status.

Runs last (file name) so that a failure here never hides another test; it
passes both alone in a fresh process and after the rest of the suite.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def GW():
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G
    import long_context_gsa_b200.workloads as W
    return G, W


def _decode_both(G, W, cfg, seed, n_max=None, t_max=None):
    x = W.decode_inputs(cfg, device="cuda", own_len=5, seed=seed, n_max=n_max, t_max=t_max)
    B, hq, d = x["q"].shape
    desc = G.make_desc(B, hq, cfg.hkv, d, cfg.chunk, x["gist_k"].shape[2], x["raw_k"].shape[2], cfg.topk,
                       cfg.exclude, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device="cuda")
    G.gsa_workspace_init(ws)
    ref = dict(out=torch.empty((B, hq, d), dtype=torch.float32, device="cuda"),
               lse=torch.empty((B, hq), dtype=torch.float32, device="cuda"),
               sel=torch.empty((B, hq, cfg.topk), dtype=torch.int32, device="cuda"))
    G.gsa_decode(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                 ref["out"], ref["lse"], ref["sel"], None, ws)
    got = dict(out=torch.full((B, hq, d), float("nan"), dtype=torch.float32, device="cuda"),
               lse=torch.full((B, hq), float("nan"), dtype=torch.float32, device="cuda"),
               sel=torch.full((B, hq, cfg.topk), -5, dtype=torch.int32, device="cuda"))
    G.gsa_decode_noalloc(desc, x["q"], x["gist_k"], x["gist_v"], x["raw_k"], x["raw_v"], x["n_gists"], x["own_len"],
                         got["out"], got["lse"], got["sel"], None)
    torch.cuda.synchronize()
    assert G.gsa_workspace_status(ws) == 0
    assert G.gsa_noalloc_status() == 0, "device status flags set by the scratch-free call"
    return ref, got


def _compare(ref, got, what):
    assert torch.isfinite(got["out"]).all(), f"{what}: output not written"
    err = (got["out"] - ref["out"]).abs().max().item()
    assert err <= 2e-3, f"{what}: max abs err {err}"
    lerr = (got["lse"] - ref["lse"]).abs().max().item()
    assert lerr <= 2e-3, f"{what}: lse max abs err {lerr}"
    assert torch.equal(torch.sort(got["sel"], -1).values, torch.sort(ref["sel"], -1).values), f"{what}: selection"


SHAPES = {
    # Llama-3.2-1B head layout (d = 64, GQA 4), default set and exclude-unselected
    "llama_default": lambda W: W.scaled(W.LLAMA_8X, batch=4, context=1024 * 8),
    "llama_exclude": lambda W: W.scaled(W.LLAMA_8X, batch=4, context=1024 * 8, exclude=True),
    # Qwen2-7B head layout (d = 128, GQA 7)
    "qwen_d128_gqa7": lambda W: W.scaled(W.QWEN_16X, batch=2, context=512 * 16),
}


@pytest.mark.parametrize("shape", list(SHAPES))
def test_noalloc_matches_decode_on_two_calls_in_a_row(GW, shape):
    G, W = GW
    cfg = SHAPES[shape](W)
    for call, seed in enumerate((101, 202)):  # two calls in a row, different inputs
        ref, got = _decode_both(G, W, cfg, seed)
        _compare(ref, got, f"{shape} call {call}")


def test_noalloc_near_its_scratch_limit(GW):
    """A problem whose workspace fills the scratch array to within a few KB,
    so the last bytes of the array are in use."""
    G, W = GW
    base = W.scaled(W.QWEN_16X, batch=16, context=64 * 16, topk=16)
    lim = 32 << 20

    def ws_bytes(n):
        return G.gsa_workspace_bytes(G.make_desc(base.batch, base.hq, base.hkv, base.d, base.chunk, n,
                                                 n * base.chunk + base.chunk, base.topk, False, 0.0, G.GSA_BF16,
                                                 G.GSA_F32), G.GSA_OP_DECODE)
    lo, hi = 1, 1 << 16
    while lo < hi:  # largest gist capacity whose workspace still fits
        mid = (lo + hi + 1) // 2
        lo, hi = (mid, hi) if ws_bytes(mid) <= lim else (lo, mid - 1)
    n_max = lo
    assert lim - 64 * 1024 < ws_bytes(n_max) <= lim < ws_bytes(n_max + 1)
    cfg = W.scaled(base, context=n_max * base.chunk)
    for call, seed in enumerate((303, 404)):
        ref, got = _decode_both(G, W, cfg, seed, n_max=n_max, t_max=n_max * base.chunk + base.chunk)
        _compare(ref, got, f"near-limit call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch(GW):
    """The C entry point refuses, before enqueueing anything, a problem whose
    workspace would not fit the scratch array (called through ctypes
    directly: the binding's own size checks would stop these tiny buffers
    first)."""
    import ctypes as C
    G, _ = GW
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(4, dtype=torch.int32, device="cuda")
    o = torch.zeros(64, dtype=torch.float32, device="cuda")
    big = G.make_desc(16, 32, 8, 64, 8, 1 << 20, (1 << 20) * 8, 64, False, 0.0, G.GSA_BF16, G.GSA_F32)
    assert G.gsa_workspace_bytes(big, G.GSA_OP_DECODE) > (32 << 20)
    st = G.load().gsa_decode_noalloc(C.byref(big), t.data_ptr(), t.data_ptr(), t.data_ptr(), t.data_ptr(),
                                     t.data_ptr(), i.data_ptr(), i.data_ptr(), o.data_ptr(), None, None, None, None)
    assert st == G.GSA_ERR_WORKSPACE
