"""Float64 CPU oracle for Gist Sparse Attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product package
(``long_context_gsa_b200``) never imports it and shares no code with it.

The arithmetic lives in ``gsa_oracle.c`` (plain C, float64, scalar loops);
this module only compiles it with gcc, mirrors its argument blocks with
ctypes and marshals numpy arrays.  Inputs are passed in their storage type:
``float32`` arrays, or ``uint16`` arrays holding bfloat16 bit patterns, which
the C code widens exactly.

Layouts (row-major):
  decode   q [B,Hq,d]; gist_k/gist_v [B,Hkv,n_max,d]; raw_k/raw_v [B,Hkv,t_max,d];
           meta_k/meta_v [B,Hkv,m_max,d]; n_gists, own_len int32 [B]
  prefill  q_raw [B,Hq,L,d]; k_raw/v_raw [B,Hkv,L,d] with L = n_chunks*chunk;
           q_gist [B,Hq,N,d]; k_gist/v_gist [B,Hkv,N,d]
Query head h reads kv head h // (Hq // Hkv).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import sys
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "gsa_oracle.c"
_BUILD = _HERE / "_build"
_LIB = _BUILD / "libgsa_oracle.so"

F32, BF16 = 0, 1
TOK_RAW, TOK_GIST, TOK_META = 0, 1, 2

_vp = C.c_void_p
_ip = C.POINTER(C.c_int32)
_lp = C.POINTER(C.c_int64)
_dp = C.POINTER(C.c_double)


class _DecodeArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_max", C.c_int32), ("t_max", C.c_int32), ("topk", C.c_int32), ("exclude", C.c_int32), ("dtype", C.c_int32),
        ("scale", C.c_double),
        ("q", _vp), ("gist_k", _vp), ("gist_v", _vp), ("raw_k", _vp), ("raw_v", _vp),
        ("n_gists", _ip), ("own_len", _ip),
        ("n_rows", C.c_int32), ("rows", _ip), ("sel_in", _ip),
        ("out", _dp), ("lse", _dp), ("sel_out", _ip), ("sel_score", _dp), ("scores", _dp),
        ("set_cap", C.c_int32), ("set_n", _ip), ("set_kind", _ip), ("set_idx", _ip), ("set_w", _dp),
        ("n_threads", C.c_int32),
    ]


class _HgsaArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_max", C.c_int32), ("t_max", C.c_int32), ("m_max", C.c_int32), ("topk", C.c_int32),
        ("exclude", C.c_int32), ("dtype", C.c_int32), ("group", C.c_int32), ("topk_meta", C.c_int32),
        ("scale", C.c_double),
        ("q", _vp), ("meta_k", _vp), ("meta_v", _vp), ("gist_k", _vp), ("gist_v", _vp), ("raw_k", _vp), ("raw_v", _vp),
        ("n_gists", _ip), ("own_len", _ip),
        ("n_rows", C.c_int32), ("rows", _ip), ("meta_sel_in", _ip), ("sel_in", _ip),
        ("out", _dp), ("lse", _dp), ("meta_sel_out", _ip), ("sel_out", _ip),
        ("meta_scores", _dp), ("cand_scores", _dp),
        ("set_cap", C.c_int32), ("set_n", _ip), ("set_kind", _ip), ("set_idx", _ip), ("set_w", _dp),
        ("n_threads", C.c_int32),
    ]


class _DecodeBwdArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_max", C.c_int32), ("t_max", C.c_int32), ("topk", C.c_int32), ("exclude", C.c_int32),
        ("dtype", C.c_int32), ("scale", C.c_double),
        ("q", _vp), ("gist_k", _vp), ("gist_v", _vp), ("raw_k", _vp), ("raw_v", _vp),
        ("n_gists", _ip), ("own_len", _ip), ("sel_in", _ip), ("d_out", _dp), ("d_q", _dp),
        ("d_gist_k", _dp), ("d_gist_v", _dp), ("d_raw_k", _dp), ("d_raw_v", _dp),
    ]


class _GistStepArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_max", C.c_int32), ("t_max", C.c_int32), ("dtype", C.c_int32), ("scale", C.c_double),
        ("q", _vp), ("k_new", _vp), ("v_new", _vp), ("gist_k", _vp), ("gist_v", _vp), ("raw_k", _vp),
        ("raw_v", _vp), ("n_gists", _ip), ("own_len", _ip), ("out", _dp), ("lse", _dp), ("n_threads", C.c_int32),
    ]


class _Hgsa2Args(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_max", C.c_int32), ("t_max", C.c_int32), ("m1_max", C.c_int32), ("m2_max", C.c_int32),
        ("group1", C.c_int32), ("group2", C.c_int32), ("topk2", C.c_int32), ("topk1", C.c_int32),
        ("topk", C.c_int32), ("exclude", C.c_int32), ("dtype", C.c_int32), ("scale", C.c_double),
        ("q", _vp), ("meta2_k", _vp), ("meta2_v", _vp), ("meta_k", _vp), ("meta_v", _vp), ("gist_k", _vp),
        ("gist_v", _vp), ("raw_k", _vp), ("raw_v", _vp), ("n_gists", _ip), ("own_len", _ip),
        ("n_rows", C.c_int32), ("rows", _ip), ("meta2_sel_in", _ip), ("meta_sel_in", _ip), ("sel_in", _ip),
        ("out", _dp), ("lse", _dp), ("meta2_sel_out", _ip), ("meta_sel_out", _ip), ("sel_out", _ip),
        ("meta2_scores", _dp), ("meta_cand_scores", _dp), ("cand_scores", _dp),
        ("set_cap", C.c_int32), ("set_n", _ip), ("set_kind", _ip), ("set_idx", _ip), ("set_w", _dp),
        ("n_threads", C.c_int32),
    ]


class _PrefillArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32), ("chunk", C.c_int32),
        ("n_chunks", C.c_int32), ("topk", C.c_int32), ("exclude", C.c_int32), ("dtype", C.c_int32),
        ("scale", C.c_double),
        ("q_raw", _vp), ("k_raw", _vp), ("v_raw", _vp), ("q_gist", _vp), ("k_gist", _vp), ("v_gist", _vp),
        ("n_rows", C.c_int32), ("rows", _lp), ("sel_in", _ip),
        ("out", _dp), ("lse", _dp), ("sel_out", _ip), ("sel_score", _dp),
        ("set_cap", C.c_int32), ("set_n", _ip), ("set_kind", _ip), ("set_idx", _ip), ("set_w", _dp),
        ("n_threads", C.c_int32),
    ]


def build(src: Path | None = None, out: Path | None = None, extra_flags: tuple[str, ...] = ()) -> Path:
    """Compile the oracle with gcc (``-O2``, no fast-math) and return the .so path."""
    src = Path(src or _SRC)
    out = Path(out or _LIB)
    out.parent.mkdir(parents=True, exist_ok=True)
    if out.exists() and out.stat().st_mtime >= src.stat().st_mtime and not extra_flags:
        return out
    tmp = out.with_suffix(f".{os.getpid()}.tmp")
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           *extra_flags, str(src), "-o", str(tmp), "-lm", "-lpthread"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes front end over one compiled oracle library."""

    def __init__(self, lib_path: Path | None = None):
        path = Path(lib_path) if lib_path else build()
        self.path = path
        self.lib = C.CDLL(str(path))
        for name, argt in (("gsa_oracle_decode", _DecodeArgs), ("gsa_oracle_hgsa", _HgsaArgs),
                           ("gsa_oracle_hgsa2", _Hgsa2Args), ("gsa_oracle_decode_backward", _DecodeBwdArgs),
                           ("gsa_oracle_gist_step", _GistStepArgs),
                           ("gsa_oracle_prefill", _PrefillArgs)):
            fn = getattr(self.lib, name)
            fn.argtypes = [C.POINTER(argt)]
            fn.restype = C.c_int
        self.lib.gsa_oracle_default_threads.restype = C.c_int
        self.lib.gsa_oracle_topk.argtypes = [_dp, _ip, C.c_int64, C.c_int32, C.c_int32, _ip, _dp]
        self.lib.gsa_oracle_topk.restype = C.c_int
        self.lib.gsa_oracle_topp.argtypes = [_dp, _ip, C.c_int64, C.c_int32, C.c_int32, C.c_double, _ip, _dp, _ip,
                                             _dp, _dp]
        self.lib.gsa_oracle_topp.restype = C.c_int

    def default_threads(self) -> int:
        return int(self.lib.gsa_oracle_default_threads())

    # ------------------------------------------------------------------ decode
    def decode(self, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, *, chunk, topk, exclude=False,
               scale=0.0, rows=None, sel_in=None, want_scores=False, set_cap=0, n_threads=0):
        """Flat GSA decode for the given rows (row id = b*Hq + h; None = all)."""
        dtype, arrs = _storage(q, gist_k, gist_v, raw_k, raw_v)
        q, gist_k, gist_v, raw_k, raw_v = arrs
        B, Hq, d = q.shape
        _, Hkv, n_max, _ = gist_k.shape
        t_max = raw_k.shape[2]
        _check_shapes(gist_k, (B, Hkv, n_max, d), gist_v, raw_k, raw_v, t_max)
        n_gists, own_len = _i32(n_gists), _i32(own_len)
        rows_a, n_rows = _rows32(rows, B * Hq)
        sel_in_a = None if sel_in is None else _i32(sel_in).reshape(n_rows, topk)
        res = _alloc(n_rows, d, topk, set_cap, scores=n_max if want_scores else 0)
        a = _DecodeArgs(B, Hq, Hkv, d, chunk, n_max, t_max, topk, int(bool(exclude)), dtype, float(scale),
                        _ptr(q), _ptr(gist_k), _ptr(gist_v), _ptr(raw_k), _ptr(raw_v),
                        _ip_(n_gists), _ip_(own_len), n_rows, _ip_(rows_a), _ip_(sel_in_a),
                        _dp_(res["out"]), _dp_(res["lse"]), _ip_(res["sel"]), _dp_(res["sel_score"]),
                        _dp_(res.get("scores")), set_cap, _ip_(res.get("set_n")), _ip_(res.get("set_kind")),
                        _ip_(res.get("set_idx")), _dp_(res.get("set_w")), n_threads)
        _ok(self.lib.gsa_oracle_decode(C.byref(a)), "decode")
        return res

    def multiquery_select(self, q, gist_k, *, topk, scale=0.0, rows=None, n_threads=0):
        """Top-k gists of every query against one shared, complete gist cache
        (KV reuse).  q [B, Hq, Q, d]; query head h reads kv head h / (Hq/Hkv);
        gist_k [B, Hkv, N, d].  These are the decode oracle's scoring and
        selection steps with the Q queries of head h taken as query heads
        h*Q .. h*Q+Q-1 of a group of Q*Hq/Hkv heads (so they read the same
        kv head h / (Hq/Hkv)), N completed gists and no raw rows.  Row id
        (b*Hq + h)*Q + i.  Returns the decode result dict (sel in rank order,
        sel_score, scores; out / lse are those of the compression-only set)."""
        dtype, arrs = _storage(q, gist_k)
        q, gist_k = arrs
        B, Hq, Q, d = q.shape
        _, Hkv, N, _ = gist_k.shape
        no_raw = np.zeros((B, Hkv, N, d), dtype=gist_k.dtype)
        return self.decode(q.reshape(B, Hq * Q, d), gist_k, gist_k, no_raw, no_raw, np.full(B, N, np.int32),
                           np.zeros(B, np.int32), chunk=1, topk=topk, scale=scale, rows=rows, want_scores=True,
                           n_threads=n_threads)

    def decode_backward(self, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, sel_in, d_out, *, chunk, topk,
                        exclude=False, scale=0.0):
        """Gradients of sum(d_out * out) of a decode step with the given
        (fixed) selection: d_q [B, Hq, d]; d_gist_k/v, d_raw_k/v shaped like
        their inputs (float64)."""
        dtype, arrs = _storage(q, gist_k, gist_v, raw_k, raw_v)
        q, gist_k, gist_v, raw_k, raw_v = arrs
        B, Hq, d = q.shape
        _, Hkv, n_max, _ = gist_k.shape
        t_max = raw_k.shape[2]
        _check_shapes(gist_k, (B, Hkv, n_max, d), gist_v, raw_k, raw_v, t_max)
        sel = _i32(sel_in).reshape(B * Hq, topk) if topk else None
        g = np.ascontiguousarray(d_out, dtype=np.float64).reshape(B * Hq, d)
        res = {"d_q": np.zeros((B, Hq, d)), "d_gist_k": np.zeros((B, Hkv, n_max, d)),
               "d_gist_v": np.zeros((B, Hkv, n_max, d)), "d_raw_k": np.zeros((B, Hkv, t_max, d)),
               "d_raw_v": np.zeros((B, Hkv, t_max, d))}
        n_gists, own_len = _i32(n_gists), _i32(own_len)
        a = _DecodeBwdArgs(B, Hq, Hkv, d, chunk, n_max, t_max, topk, int(bool(exclude)), dtype, float(scale),
                           _ptr(q), _ptr(gist_k), _ptr(gist_v), _ptr(raw_k), _ptr(raw_v), _ip_(n_gists),
                           _ip_(own_len), _ip_(sel), g.ctypes.data_as(_dp), _dp_(res["d_q"]), _dp_(res["d_gist_k"]),
                           _dp_(res["d_gist_v"]), _dp_(res["d_raw_k"]), _dp_(res["d_raw_v"]))
        _ok(self.lib.gsa_oracle_decode_backward(C.byref(a)), "decode_backward")
        return res

    def gist_step(self, q, k_new, v_new, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, *, chunk, scale=0.0,
                  n_threads=0):
        """Gist-position step at chunk completion: q [B, Hq, d] attends the
        gists 0..N-1, the own chunk's raw rows and itself (k_new / v_new
        [B, Hkv, d]).  Returns {"out": [B*Hq, d], "lse": [B*Hq]}."""
        dtype, arrs = _storage(q, k_new, v_new, gist_k, gist_v, raw_k, raw_v)
        q, k_new, v_new, gist_k, gist_v, raw_k, raw_v = arrs
        B, Hq, d = q.shape
        _, Hkv, n_max, _ = gist_k.shape
        t_max = raw_k.shape[2]
        _check_shapes(gist_k, (B, Hkv, n_max, d), gist_v, raw_k, raw_v, t_max)
        if k_new.shape != (B, Hkv, d) or v_new.shape != (B, Hkv, d):
            raise ValueError("k_new / v_new shape")
        res = {"out": np.zeros((B * Hq, d)), "lse": np.zeros(B * Hq)}
        n_gists, own_len = _i32(n_gists), _i32(own_len)
        a = _GistStepArgs(B, Hq, Hkv, d, chunk, n_max, t_max, dtype, float(scale), _ptr(q), _ptr(k_new), _ptr(v_new),
                          _ptr(gist_k), _ptr(gist_v), _ptr(raw_k), _ptr(raw_v), _ip_(n_gists), _ip_(own_len),
                          _dp_(res["out"]), _dp_(res["lse"]), n_threads)
        _ok(self.lib.gsa_oracle_gist_step(C.byref(a)), "gist_step")
        return res

    # -------------------------------------------------------------------- topk
    def topk(self, scores, n_valid, k):
        """Selection step alone on given scores [rows, stride] (float64 compare):
        (sel [rows, k] ascending index, -1 padded; sel_score, -inf padded)."""
        s = np.ascontiguousarray(scores, dtype=np.float64)
        rows, stride = s.shape
        n = _i32(n_valid)
        if n.shape != (rows,):
            raise ValueError("n_valid shape")
        sel = np.full((rows, k), -1, np.int32)
        ssc = np.zeros((rows, k))
        _ok(self.lib.gsa_oracle_topk(s.ctypes.data_as(_dp), _ip_(n), rows, stride, k, _ip_(sel), _dp_(ssc)), "topk")
        return sel, ssc

    def topp(self, scores, n_valid, k, top_p):
        """Top-p (nucleus) selection on given scores [rows, stride]: the shortest
        rank-order prefix with softmax mass >= top_p, 1..k entries.  Returns
        dict(sel, sel_score, count, mass_lo, mass_hi)."""
        s = np.ascontiguousarray(scores, dtype=np.float64)
        rows, stride = s.shape
        n = _i32(n_valid)
        if n.shape != (rows,):
            raise ValueError("n_valid shape")
        res = {"sel": np.full((rows, k), -1, np.int32), "sel_score": np.zeros((rows, k)),
               "count": np.zeros(rows, np.int32), "mass_lo": np.zeros(rows), "mass_hi": np.zeros(rows)}
        _ok(self.lib.gsa_oracle_topp(s.ctypes.data_as(_dp), _ip_(n), rows, stride, k, float(top_p), _ip_(res["sel"]),
                                     _dp_(res["sel_score"]), _ip_(res["count"]), _dp_(res["mass_lo"]),
                                     _dp_(res["mass_hi"])), "topp")
        return res

    # -------------------------------------------------------------------- hgsa
    def hgsa(self, q, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, *, chunk, group,
             topk_meta, topk, exclude=False, scale=0.0, rows=None, meta_sel_in=None, sel_in=None,
             want_scores=False, set_cap=0, n_threads=0):
        """H-GSA decode (one meta level) for the given rows."""
        dtype, arrs = _storage(q, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v)
        q, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v = arrs
        B, Hq, d = q.shape
        _, Hkv, n_max, _ = gist_k.shape
        m_max, t_max = meta_k.shape[2], raw_k.shape[2]
        _check_shapes(gist_k, (B, Hkv, n_max, d), gist_v, raw_k, raw_v, t_max)
        if meta_k.shape != (B, Hkv, m_max, d) or meta_v.shape != meta_k.shape:
            raise ValueError("meta_k/meta_v shape")
        n_gists, own_len = _i32(n_gists), _i32(own_len)
        rows_a, n_rows = _rows32(rows, B * Hq)
        msel = None if meta_sel_in is None else _i32(meta_sel_in).reshape(n_rows, topk_meta)
        sel = None if sel_in is None else _i32(sel_in).reshape(n_rows, topk)
        res = _alloc(n_rows, d, topk, set_cap)
        res["meta_sel"] = np.full((n_rows, topk_meta), -1, np.int32)
        if want_scores:
            res["meta_scores"] = np.zeros((n_rows, m_max))
            res["cand_scores"] = np.zeros((n_rows, n_max))
        a = _HgsaArgs(B, Hq, Hkv, d, chunk, n_max, t_max, m_max, topk, int(bool(exclude)), dtype, group,
                      topk_meta, float(scale), _ptr(q), _ptr(meta_k), _ptr(meta_v), _ptr(gist_k), _ptr(gist_v),
                      _ptr(raw_k), _ptr(raw_v), _ip_(n_gists), _ip_(own_len), n_rows, _ip_(rows_a), _ip_(msel),
                      _ip_(sel), _dp_(res["out"]), _dp_(res["lse"]), _ip_(res["meta_sel"]), _ip_(res["sel"]),
                      _dp_(res.get("meta_scores")), _dp_(res.get("cand_scores")), set_cap,
                      _ip_(res.get("set_n")), _ip_(res.get("set_kind")), _ip_(res.get("set_idx")),
                      _dp_(res.get("set_w")), n_threads)
        _ok(self.lib.gsa_oracle_hgsa(C.byref(a)), "hgsa")
        return res

    def hgsa2(self, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, *,
              chunk, group1, group2, topk2, topk1, topk, exclude=False, scale=0.0, rows=None, meta2_sel_in=None,
              meta_sel_in=None, sel_in=None, want_scores=False, set_cap=0, n_threads=0):
        """H-GSA decode with two meta levels for the given rows."""
        dtype, arrs = _storage(q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v)
        q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v = arrs
        B, Hq, d = q.shape
        _, Hkv, n_max, _ = gist_k.shape
        m1_max, m2_max, t_max = meta_k.shape[2], meta2_k.shape[2], raw_k.shape[2]
        _check_shapes(gist_k, (B, Hkv, n_max, d), gist_v, raw_k, raw_v, t_max)
        if meta_k.shape != (B, Hkv, m1_max, d) or meta_v.shape != meta_k.shape:
            raise ValueError("meta_k/meta_v shape")
        if meta2_k.shape != (B, Hkv, m2_max, d) or meta2_v.shape != meta2_k.shape:
            raise ValueError("meta2_k/meta2_v shape")
        n_gists, own_len = _i32(n_gists), _i32(own_len)
        rows_a, n_rows = _rows32(rows, B * Hq)
        m2s = None if meta2_sel_in is None else _i32(meta2_sel_in).reshape(n_rows, topk2)
        m1s = None if meta_sel_in is None else _i32(meta_sel_in).reshape(n_rows, topk1)
        sel = None if sel_in is None else _i32(sel_in).reshape(n_rows, topk)
        res = _alloc(n_rows, d, topk, set_cap)
        res["meta2_sel"] = np.full((n_rows, topk2), -1, np.int32)
        res["meta_sel"] = np.full((n_rows, topk1), -1, np.int32)
        if want_scores:
            res["meta2_scores"] = np.zeros((n_rows, m2_max))
            res["meta_cand_scores"] = np.zeros((n_rows, m1_max))
            res["cand_scores"] = np.zeros((n_rows, n_max))
        a = _Hgsa2Args(B, Hq, Hkv, d, chunk, n_max, t_max, m1_max, m2_max, group1, group2, topk2, topk1, topk,
                       int(bool(exclude)), dtype, float(scale), _ptr(q), _ptr(meta2_k), _ptr(meta2_v), _ptr(meta_k),
                       _ptr(meta_v), _ptr(gist_k), _ptr(gist_v), _ptr(raw_k), _ptr(raw_v), _ip_(n_gists),
                       _ip_(own_len), n_rows, _ip_(rows_a), _ip_(m2s), _ip_(m1s), _ip_(sel), _dp_(res["out"]),
                       _dp_(res["lse"]), _ip_(res["meta2_sel"]), _ip_(res["meta_sel"]), _ip_(res["sel"]),
                       _dp_(res.get("meta2_scores")), _dp_(res.get("meta_cand_scores")), _dp_(res.get("cand_scores")),
                       set_cap, _ip_(res.get("set_n")), _ip_(res.get("set_kind")), _ip_(res.get("set_idx")),
                       _dp_(res.get("set_w")), n_threads)
        _ok(self.lib.gsa_oracle_hgsa2(C.byref(a)), "hgsa2")
        return res

    # ----------------------------------------------------------------- prefill
    def prefill(self, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist, *, chunk, topk, exclude=False, scale=0.0,
                rows=None, sel_in=None, set_cap=0, n_threads=0):
        """Causal prefill rows.  Row id = (b*Hq + h) * (L + N) + pos, where
        pos < L is a raw position and pos = L + m is gist m."""
        dtype, arrs = _storage(q_raw, k_raw, v_raw, q_gist, k_gist, v_gist)
        q_raw, k_raw, v_raw, q_gist, k_gist, v_gist = arrs
        B, Hq, L, d = q_raw.shape
        Hkv, N = k_raw.shape[1], k_gist.shape[2]
        if L != N * chunk:
            raise ValueError("raw length must be n_chunks * chunk")
        if k_raw.shape != (B, Hkv, L, d) or v_raw.shape != k_raw.shape:
            raise ValueError("k_raw/v_raw shape")
        if q_gist.shape != (B, Hq, N, d) or k_gist.shape != (B, Hkv, N, d) or v_gist.shape != k_gist.shape:
            raise ValueError("gist array shape")
        total = B * Hq * (L + N)
        if rows is None:
            rows_a, n_rows = None, total
        else:
            rows_a = np.ascontiguousarray(rows, dtype=np.int64)
            n_rows = rows_a.size
        sel = None if sel_in is None else _i32(sel_in).reshape(n_rows, topk)
        res = _alloc(n_rows, d, topk, set_cap)
        a = _PrefillArgs(B, Hq, Hkv, d, chunk, N, topk, int(bool(exclude)), dtype, float(scale),
                         _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(q_gist), _ptr(k_gist), _ptr(v_gist),
                         n_rows, None if rows_a is None else rows_a.ctypes.data_as(_lp), _ip_(sel),
                         _dp_(res["out"]), _dp_(res["lse"]), _ip_(res["sel"]), _dp_(res["sel_score"]), set_cap,
                         _ip_(res.get("set_n")), _ip_(res.get("set_kind")), _ip_(res.get("set_idx")),
                         _dp_(res.get("set_w")), n_threads)
        _ok(self.lib.gsa_oracle_prefill(C.byref(a)), "prefill")
        return res


# ---------------------------------------------------------------- marshalling
def _storage(*arrs):
    """All arrays float32, or all uint16 (bf16 bits); returns (dtype code, contiguous arrays)."""
    kinds = {a.dtype for a in arrs}
    if kinds == {np.dtype(np.float32)}:
        code = F32
    elif kinds <= {np.dtype(np.uint16), np.dtype(np.int16)}:
        code = BF16
    else:
        raise TypeError(f"oracle inputs must be all float32 or all bf16 bits (uint16), got {kinds}")
    return code, [np.ascontiguousarray(a) for a in arrs]


def _check_shapes(gist_k, want, gist_v, raw_k, raw_v, t_max):
    B, Hkv, _, d = want
    if gist_k.shape != want or gist_v.shape != want:
        raise ValueError("gist_k/gist_v shape")
    if raw_k.shape != (B, Hkv, t_max, d) or raw_v.shape != raw_k.shape:
        raise ValueError("raw_k/raw_v shape")


def _alloc(n_rows, d, topk, set_cap, scores=0):
    res = {"out": np.zeros((n_rows, d)), "lse": np.zeros(n_rows),
           "sel": np.full((n_rows, topk), -1, np.int32), "sel_score": np.zeros((n_rows, topk))}
    if scores:
        res["scores"] = np.zeros((n_rows, scores))
    if set_cap:
        res["set_n"] = np.zeros(n_rows, np.int32)
        res["set_kind"] = np.full((n_rows, set_cap), -1, np.int32)
        res["set_idx"] = np.full((n_rows, set_cap), -1, np.int32)
        res["set_w"] = np.zeros((n_rows, set_cap))
    return res


def _rows32(rows, total):
    if rows is None:
        return None, total
    r = np.ascontiguousarray(rows, dtype=np.int32)
    return r, r.size


def _i32(x):
    return np.ascontiguousarray(x, dtype=np.int32)


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def _ip_(a):
    return None if a is None else a.ctypes.data_as(_ip)


def _dp_(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _ok(st, what):
    if st != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {st})")


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from the committed source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even) and return the bit patterns.

    Used only to build small bf16 test inputs on the host.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16).view(np.float32)


if __name__ == "__main__":  # pragma: no cover
    print(build())
    sys.exit(0)
