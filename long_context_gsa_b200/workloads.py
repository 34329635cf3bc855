"""Seeded synthetic inputs shaped like the GSA pages' workloads.

This module only draws random tensors; it contains none of the method's
arithmetic (no scoring, selection or attention).  Both the CUDA path and the
float64 oracle are fed from it, so each parity test compares the two on
exactly the same values.

The pages (gist.science explainers of "Forget, Then Recall ... Gist Sparse
Attention") evaluate Qwen2-7B and Llama3.2-1B at 8x-32x compression on
LongBench and five RAG benchmarks.  No dataset or trained weight is used
here: the head layouts and compression ratios are kept, token contents are
Gaussian, and a "relevant" chunk is planted per query head so that selection
has something to find.  Gist keys/values stand in for trained gist tokens as
the mean of their chunk's raw rows plus Gaussian noise (std 0.5); meta-gists
likewise from their children.

Noise parameters are standard deviations.  Every generator takes an explicit
seed and device; the same (seed, device) always gives the same tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    hq: int
    hkv: int
    d: int
    chunk: int
    context: int            # raw tokens before the current one (multiple of chunk)
    topk: int
    dtype: str = "bf16"
    kv_std: float = 1.0
    exclude: bool = False
    # H-GSA
    group: int = 0          # gists per meta-gist; 0 = flat GSA
    topk_meta: int = 0
    group2: int = 0         # meta-gists per level-2 meta-gist; 0 = one meta level
    topk_meta2: int = 0
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n_gists(self) -> int:
        return self.context // self.chunk

    @property
    def head_queries(self) -> int:
        return self.batch * self.hq


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    batch: int
    hq: int
    hkv: int
    d: int
    chunk: int
    n_chunks: int
    topk: int
    dtype: str = "bf16"
    exclude: bool = False
    seed: int = 0

    @property
    def length(self) -> int:
        return self.n_chunks * self.chunk


@dataclass(frozen=True)
class MultiQueryConfig:
    """Several queries routed over one document's complete gist cache (KV
    reuse): `queries` query rows per (document, query head)."""
    name: str
    batch: int
    hq: int
    hkv: int
    d: int
    n_gists: int
    queries: int
    topk: int
    dtype: str = "bf16"
    seed: int = 0

    @property
    def flops(self) -> int:
        return 2 * self.batch * self.hq * self.queries * self.n_gists * self.d


# The five workloads: a tiny fp32 single-head decode stepped 64 times, two
# flat decodes at 8x / 16x compression, an H-GSA decode at 32x and a causal
# prefill.  Seeds are fixed per workload.
PR1 = DecodeConfig("pr1_tiny_f32", 1, 1, 1, 64, 16, 4096, 8, "f32", seed=20260001, extra={"steps": 64})
LLAMA_8X = DecodeConfig("llama1b_8x", 16, 32, 8, 64, 8, 32768, 64, "bf16", seed=20260002)
QWEN_16X = DecodeConfig("qwen7b_16x", 4, 28, 4, 128, 16, 131072, 128, "bf16", kv_std=1 / math.sqrt(128),
                        seed=20260003)
QWEN_16X_EXCL = DecodeConfig("qwen7b_16x_excl", 4, 28, 4, 128, 16, 131072, 128, "bf16", kv_std=1 / math.sqrt(128),
                             exclude=True, seed=20260003)
HGSA_32X = DecodeConfig("hgsa_32x", 2, 32, 8, 128, 32, 524288, 64, "bf16", group=16, topk_meta=32, seed=20260004)
# H-GSA with a second meta level over the same 512K context: 16 level-1
# meta-gists per level-2 meta-gist (64 of them); keep 8 level-2 groups, then
# 32 of their 128 level-1 children, then 64 of those 512 gists.
HGSA2_32X = DecodeConfig("hgsa2_32x", 2, 32, 8, 128, 32, 524288, 64, "bf16", group=16, topk_meta=32, group2=16,
                         topk_meta2=8, seed=20260006)
PREFILL_32K = PrefillConfig("prefill_32k", 1, 28, 4, 128, 16, 2048, 16, "bf16", seed=20260005)
# The same causal prefill with the Llama-3.2-1B head layout (32 query / 8 kv
# heads, d = 64) at 8x compression, with the decode workload's top-64: 4096
# chunks of 8 over 32K tokens.
PREFILL_LLAMA_32K = PrefillConfig("prefill_llama1b_32k", 1, 32, 8, 64, 8, 4096, 64, "bf16", seed=20260008)
# KV reuse: a 128K-token document compressed 16x (8192 gists) shared by 4096
# query rows per head (Qwen2-7B head layout), top-16 routing per query.
KVREUSE_QWEN = MultiQueryConfig("kvreuse_qwen7b", 1, 28, 4, 128, 8192, 4096, 16, seed=20260007)

CONFIGS = {c.name: c for c in (PR1, LLAMA_8X, QWEN_16X, QWEN_16X_EXCL, HGSA_32X, HGSA2_32X, PREFILL_32K,
                               PREFILL_LLAMA_32K, KVREUSE_QWEN)}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device, std=1.0):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x.mul_(std) if std != 1.0 else x


def _plant(keys, kvh_rows, qdir, chunks, g, device, d):
    """keys[kvh_rows][chunk] <- 0.8 * qhat * sqrt(d) + N(0, 0.1^2)."""
    for row, (kv, m) in enumerate(zip(kvh_rows, chunks)):
        keys[kv, m] = 0.8 * qdir[row] * math.sqrt(d) + 0.1 * _randn((d,), g, device)


def decode_inputs(cfg: DecodeConfig, device="cpu", seed=None, own_len=1, n_max=None, t_max=None,
                  ragged=None, plant=True):
    """Flat or hierarchical decode inputs.

    Returns a dict of tensors: q [B,hq,d]; gist_k/gist_v [B,hkv,n_max,d];
    raw_k/raw_v [B,hkv,t_max,d]; n_gists/own_len int32 [B]; planted int64
    [B,hq] (the chunk planted for each head); and for H-GSA meta_k/meta_v
    [B,hkv,m_max,d].  `ragged` optionally gives per-batch gist counts
    (<= cfg.n_gists).
    """
    B, hq, hkv, d, c = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.chunk
    G = hq // hkv
    N = cfg.n_gists
    n_max = n_max or N
    t_max = t_max or (N + 1) * c
    g = _gen(device, cfg.seed if seed is None else seed)
    dt = DTYPES[cfg.dtype]
    out = {k: [] for k in ("q", "gist_k", "gist_v", "raw_k", "raw_v", "meta_k", "meta_v", "meta2_k", "meta2_v",
                           "planted")}
    counts = list(ragged) if ragged is not None else [N] * B
    for b in range(B):
        raw_k = _randn((hkv, t_max, d), g, device, cfg.kv_std)
        raw_v = _randn((hkv, t_max, d), g, device, cfg.kv_std)
        gist_k = torch.zeros((hkv, n_max, d), device=device)
        gist_v = torch.zeros((hkv, n_max, d), device=device)
        gist_k[:, :N] = raw_k[:, : N * c].reshape(hkv, N, c, d).mean(2) + _randn((hkv, N, d), g, device, 0.5)
        gist_v[:, :N] = raw_v[:, : N * c].reshape(hkv, N, c, d).mean(2) + _randn((hkv, N, d), g, device, 0.5)
        q = _randn((hq, d), g, device)
        qdir = q / q.norm(dim=-1, keepdim=True)
        nb = counts[b]
        if plant and nb > 0:
            # distinct planted chunks (for H-GSA also distinct meta groups) within each kv group
            planted = []
            for kv in range(hkv):
                if cfg.group and nb >= cfg.group:
                    M = nb // cfg.group
                    groups = torch.randperm(M, generator=g, device=device)[: min(M, G)].tolist()
                    groups = [groups[j % len(groups)] for j in range(G)]
                    offs = torch.randint(0, cfg.group, (G,), generator=g, device=device).tolist()
                    chunks = [grp * cfg.group + o for grp, o in zip(groups, offs)]
                else:
                    perm = torch.randperm(nb, generator=g, device=device)[: min(nb, G)].tolist()
                    chunks = [perm[j % len(perm)] for j in range(G)]
                _plant(gist_k, [kv] * G, qdir[kv * G:(kv + 1) * G], chunks, g, device, d)
                planted += chunks
            out["planted"].append(torch.tensor(planted, dtype=torch.int64))
        else:
            out["planted"].append(torch.full((hq,), -1, dtype=torch.int64))
        if cfg.group:
            M_cap = n_max // cfg.group
            M = N // cfg.group
            meta_k = torch.zeros((hkv, max(M_cap, 1), d), device=device)
            meta_v = torch.zeros((hkv, max(M_cap, 1), d), device=device)
            meta_k[:, :M] = gist_k[:, : M * cfg.group].reshape(hkv, M, cfg.group, d).mean(2) + _randn(
                (hkv, M, d), g, device, 0.5)
            meta_v[:, :M] = gist_v[:, : M * cfg.group].reshape(hkv, M, cfg.group, d).mean(2) + _randn(
                (hkv, M, d), g, device, 0.5)
            if plant and nb > 0:
                for kv in range(hkv):
                    for j in range(G):
                        m = int(out["planted"][-1][kv * G + j])
                        if m // cfg.group < M:
                            meta_k[kv, m // cfg.group] = 0.8 * qdir[kv * G + j] * math.sqrt(d) + 0.1 * _randn(
                                (d,), g, device)
            if cfg.group2:
                # level 2 from level 1 as level 1 from the gists; planted at every level
                M2_cap, M2 = max(M_cap // cfg.group2, 1), M // cfg.group2
                meta2_k = torch.zeros((hkv, M2_cap, d), device=device)
                meta2_v = torch.zeros((hkv, M2_cap, d), device=device)
                meta2_k[:, :M2] = meta_k[:, : M2 * cfg.group2].reshape(hkv, M2, cfg.group2, d).mean(2) + _randn(
                    (hkv, M2, d), g, device, 0.5)
                meta2_v[:, :M2] = meta_v[:, : M2 * cfg.group2].reshape(hkv, M2, cfg.group2, d).mean(2) + _randn(
                    (hkv, M2, d), g, device, 0.5)
                if plant and nb > 0:
                    for kv in range(hkv):
                        for j in range(G):
                            m2 = int(out["planted"][-1][kv * G + j]) // cfg.group // cfg.group2
                            if m2 < M2:
                                meta2_k[kv, m2] = 0.8 * qdir[kv * G + j] * math.sqrt(d) + 0.1 * _randn((d,), g, device)
                out["meta2_k"].append(meta2_k.to(dt))
                out["meta2_v"].append(meta2_v.to(dt))
            out["meta_k"].append(meta_k.to(dt))
            out["meta_v"].append(meta_v.to(dt))
        out["q"].append(q.to(dt))
        out["gist_k"].append(gist_k.to(dt))
        out["gist_v"].append(gist_v.to(dt))
        out["raw_k"].append(raw_k.to(dt))
        out["raw_v"].append(raw_v.to(dt))
        del raw_k, raw_v
    res = {k: torch.stack(v) for k, v in out.items() if v}
    res["n_gists"] = torch.tensor(counts, dtype=torch.int32, device=device)
    res["own_len"] = torch.full((B,), own_len, dtype=torch.int32, device=device)
    return res


def gist_step_inputs(cfg: DecodeConfig, device="cpu", seed=None, ragged=None, own_len=None):
    """Inputs of a gist-position step at chunk completion: the decode inputs
    with room for one more gist (n_max = N + 1) and a full own chunk
    (own_len = chunk unless given), plus the new gist's key / value
    k_new / v_new [B, hkv, d] drawn like the other gists (mean of the
    chunk's raw rows + N(0, 0.5)).  q is the gist-position query."""
    c = cfg.chunk
    x = decode_inputs(cfg, device=device, seed=seed, own_len=c if own_len is None else own_len,
                      n_max=cfg.n_gists + 1, t_max=(cfg.n_gists + 1) * c, ragged=ragged, plant=False)
    g = _gen(device, (cfg.seed if seed is None else seed) + 17)
    dt = DTYPES[cfg.dtype]
    B, hkv, d = cfg.batch, cfg.hkv, cfg.d
    k_new = torch.empty((B, hkv, d), device=device)
    v_new = torch.empty((B, hkv, d), device=device)
    for b in range(B):
        N = int(x["n_gists"][b])
        k_new[b] = x["raw_k"][b, :, N * c:(N + 1) * c].float().mean(1) + _randn((hkv, d), g, device, 0.5)
        v_new[b] = x["raw_v"][b, :, N * c:(N + 1) * c].float().mean(1) + _randn((hkv, d), g, device, 0.5)
    x["k_new"], x["v_new"] = k_new.to(dt), v_new.to(dt)
    return x


def pr1_steps(cfg: DecodeConfig = PR1, device="cpu", seed=None):
    """The tiny single-head workload stepped through its decode steps.

    Step s (0-based) has 4096 + s raw rows before the current token, so
    n_gists = (4096 + s) // 16 and own_len = s % 16 + 1; each time 16 own rows
    complete, the next gist (drawn from N(0,1)) becomes visible.  One base
    direction qhat0 is drawn; q_s = sqrt(d)*qhat0 + 0.25*N(0,I); 8 planted
    chunks among the first 256 have gist keys 0.8*qhat0*sqrt(d) + N(0,0.1^2).
    Returns (static inputs dict, list of per-step dicts with q, n_gists,
    own_len).
    """
    steps = cfg.extra.get("steps", 64)
    d, c = cfg.d, cfg.chunk
    N0 = cfg.context // c
    n_max = (cfg.context + steps) // c + 1
    t_max = n_max * c
    g = _gen(device, cfg.seed if seed is None else seed)
    raw_k = _randn((1, 1, t_max, d), g, device)
    raw_v = _randn((1, 1, t_max, d), g, device)
    gist_k = _randn((1, 1, n_max, d), g, device)
    gist_v = _randn((1, 1, n_max, d), g, device)
    q0 = _randn((d,), g, device)
    qhat = q0 / q0.norm()
    planted = torch.randperm(N0, generator=g, device=device)[:8]
    for m in planted.tolist():
        gist_k[0, 0, m] = 0.8 * qhat * math.sqrt(d) + 0.1 * _randn((d,), g, device)
    per_step = []
    for s in range(steps):
        pos = cfg.context + s
        q = (math.sqrt(d) * qhat + 0.25 * _randn((d,), g, device)).reshape(1, 1, d)
        per_step.append({"q": q, "n_gists": torch.tensor([pos // c], dtype=torch.int32, device=device),
                         "own_len": torch.tensor([pos % c + 1], dtype=torch.int32, device=device)})
    static = {"gist_k": gist_k, "gist_v": gist_v, "raw_k": raw_k, "raw_v": raw_v, "planted": planted.cpu()}
    return static, per_step


def multiquery_inputs(cfg: MultiQueryConfig, device="cpu", seed=None):
    """q [B,hq,Q,d] and gist_k [B,hkv,N,d], N(0,1); for each (document, kv
    head) every query row of its group has one planted gist (drawn among
    all N) whose key is 0.8*sqrt(d)*qhat + N(0, 0.1^2), as in the decode
    workloads, so routing has something to find."""
    B, hq, hkv, d, N, Q = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.n_gists, cfg.queries
    g = _gen(device, cfg.seed if seed is None else seed)
    dt = DTYPES[cfg.dtype]
    q = _randn((B, hq, Q, d), g, device)
    gk = _randn((B, hkv, N, d), g, device)
    G = hq // hkv
    for b in range(B):
        for kv in range(hkv):
            # a few planted gists per kv head, each aligned with one query row
            n_plant = min(N, 8)
            chunks = torch.randperm(N, generator=g, device=device)[:n_plant].tolist()
            for j, m in enumerate(chunks):
                h = kv * G + j % G
                i = int(torch.randint(0, Q, (1,), generator=g, device=device))
                qhat = q[b, h, i] / q[b, h, i].norm()
                gk[b, kv, m] = 0.8 * qhat * math.sqrt(d) + 0.1 * _randn((d,), g, device)
    return {"q": q.to(dt), "gist_k": gk.to(dt)}


def prefill_inputs(cfg: PrefillConfig, device="cpu", seed=None):
    """q_raw [B,hq,L,d]; k_raw/v_raw [B,hkv,L,d]; q_gist [B,hq,N,d];
    k_gist/v_gist [B,hkv,N,d]; all N(0,1)."""
    B, hq, hkv, d, N, L = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.n_chunks, cfg.length
    g = _gen(device, cfg.seed if seed is None else seed)
    dt = DTYPES[cfg.dtype]
    return {
        "q_raw": _randn((B, hq, L, d), g, device).to(dt),
        "k_raw": _randn((B, hkv, L, d), g, device).to(dt),
        "v_raw": _randn((B, hkv, L, d), g, device).to(dt),
        "q_gist": _randn((B, hq, N, d), g, device).to(dt),
        "k_gist": _randn((B, hkv, N, d), g, device).to(dt),
        "v_gist": _randn((B, hkv, N, d), g, device).to(dt),
    }


def scaled(cfg, **changes):
    """A copy of a config with some fields changed (small parity cases)."""
    from dataclasses import replace
    return replace(cfg, **changes)


def to_oracle(t: torch.Tensor):
    """Host numpy view for the oracle: float32 as is, bf16 as uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype in (torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)
