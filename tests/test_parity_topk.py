"""Top-k chunk selection alone on the GPU (gsa_topk_select) against the
oracle's selection step on the same fp32 scores.  Inputs are given scores, so
no arithmetic separates the two sides: indices and scores must match exactly,
including every exact tie (equal scores go to the lower chunk index).

The row lengths and k cover each path of the kernel: the bound path with a
sorted and with a counted candidate set, the radix select (fewer than one
full warp of entries, k above 256), the path for rows too long for registers,
k >= n, k = 0 and empty rows."""
import zlib

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

G = None


@pytest.fixture(scope="module", autouse=True)
def _setup():
    global G
    from long_context_gsa_b200 import build
    build.build_library()
    import long_context_gsa_b200 as G_
    G = G_
    torch.cuda.init()


def _scores(rng, shape, dist):
    if dist == "randn":
        return rng.standard_normal(shape).astype(np.float32)
    if dist == "ties8":  # eight levels: ties everywhere, including at the k-th place
        return (rng.integers(-4, 4, size=shape) * 0.5).astype(np.float32)
    if dist == "ties2":
        return rng.integers(0, 2, size=shape).astype(np.float32)
    if dist == "planted":  # a few clear winners over a noise floor
        s = rng.standard_normal(shape).astype(np.float32)
        s[..., rng.integers(0, shape[-1], size=5)] += 8.0
        return s
    raise ValueError(dist)


CASES = [
    # name, batch, hq, n_max, k, n_gists per batch
    ("llama_shape", 2, 32, 4096, 64, [4096, 3001]),
    ("qwen_shape", 2, 28, 8192, 128, [8192, 5000]),
    ("hgsa_children", 2, 16, 512, 64, [512, 300]),
    ("hgsa_meta", 2, 16, 1024, 32, [1024, 77]),
    ("k_above_warp_maxima", 1, 16, 2048, 200, [2048]),
    ("short_rows", 2, 8, 100, 64, [100, 65]),
    ("one_warp", 2, 8, 33, 8, [33, 32]),
    ("below_one_warp", 2, 8, 31, 8, [31, 9]),
    ("k_eq_n", 1, 8, 64, 64, [64]),
    ("k_above_n", 2, 8, 40, 64, [40, 1]),
    ("empty_rows", 2, 4, 256, 16, [0, 256]),
    ("k_above_256", 1, 4, 3000, 700, [3000]),
    ("long_rows", 1, 4, 20000, 16, [20000]),
]


@pytest.mark.parametrize("dist", ["randn", "ties8", "ties2", "planted"])
@pytest.mark.parametrize("name,B,hq,n_max,k,ng", CASES, ids=[c[0] for c in CASES])
def test_topk_matches_oracle(name, B, hq, n_max, k, ng, dist):
    rng = np.random.default_rng(zlib.crc32(f"{name}/{dist}".encode()))
    s = _scores(rng, (B, hq, n_max), dist)
    for b in range(B):
        s[b, :, ng[b]:] = np.nan  # past the row's count: never read
    dev = torch.device("cuda")
    hkv = {32: 8, 28: 4, 16: 4, 8: 2, 4: 1}[hq]
    desc = G.make_desc(B, hq, hkv, 64, 8, n_max, n_max * 8, k, False, 0.0, G.GSA_BF16, G.GSA_F32)
    ws = torch.empty(G.gsa_workspace_bytes(desc, G.GSA_OP_DECODE), dtype=torch.uint8, device=dev)
    G.gsa_workspace_init(ws)
    sel = torch.full((B, hq, max(k, 1)), -7, dtype=torch.int32, device=dev)
    ssc = torch.zeros((B, hq, max(k, 1)), dtype=torch.float32, device=dev)
    G.gsa_topk_select(desc, torch.from_numpy(s).to(dev), torch.tensor(ng, dtype=torch.int32, device=dev), sel, ssc, ws)
    torch.cuda.synchronize()
    n_valid = np.repeat(np.array(ng, np.int32), hq)
    want, want_s = oracle.get().topk(s.reshape(B * hq, n_max).astype(np.float64), n_valid, k)
    got = sel.cpu().numpy().reshape(B * hq, -1)[:, :k]
    got_s = ssc.cpu().numpy().reshape(B * hq, -1)[:, :k].astype(np.float64)
    bad = np.nonzero((got != want).any(axis=1))[0]
    assert bad.size == 0, (f"{bad.size} rows differ; first row {bad[0]}: got {got[bad[0]][:12]} "
                           f"want {want[bad[0]][:12]}" if bad.size else "")
    np.testing.assert_array_equal(got_s, want_s)
