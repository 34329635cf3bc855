"""ctypes binding of libgsa.so -- argument marshalling only.

Each function here has the name of the C entry point it calls (see
include/gsa.h for layouts and semantics), takes torch tensors, checks that
they live on the current CUDA device with the dtype and contiguity the C
ABI expects, passes their data pointers and the current (or given) stream,
and raises GsaError on a non-OK status.  No arithmetic happens here; there
is no CPU path: without the built library every call raises.
"""
from __future__ import annotations

import ctypes as C
from pathlib import Path

import torch

from .build import LIB

GSA_OK, GSA_ERR_INVALID_ARG, GSA_ERR_UNSUPPORTED, GSA_ERR_WORKSPACE, GSA_ERR_CUDA, GSA_ERR_TIMEOUT = range(6)
GSA_F32, GSA_BF16 = 0, 1
GSA_PRIOR_NONE, GSA_PRIOR_GISTS, GSA_PRIOR_HGSA, GSA_PRIOR_HGSA2 = 0, 1, 2, 3
GSA_OP_DECODE, GSA_OP_HGSA, GSA_OP_PREFILL, GSA_OP_HGSA2, GSA_OP_GIST_STEP, GSA_OP_MULTIQUERY = 0, 1, 2, 3, 4, 5
GSA_DEVERR_BAD_INDEX, GSA_DEVERR_TIMEOUT, GSA_DEVERR_CAPACITY = 1, 2, 4

EXPORTS = (
    "gsa_status_string", "gsa_version", "gsa_workspace_bytes", "gsa_workspace_init", "gsa_workspace_status",
    "gsa_score_gists", "gsa_topk_select", "gsa_topp_select", "gsa_unfold_attend", "gsa_decode", "hgsa_select",
    "hgsa_decode", "hgsa2_select", "hgsa2_decode", "gsa_decode_backward", "gsa_gist_step", "gsa_multiquery_select", "gsa_prefill_score", "gsa_prefill_attend", "gsa_prefill",
    "gsa_decode_noalloc", "gsa_noalloc_status", "gsa_score_select",
)


class GsaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg}")
        self.status = status


class gsa_desc(C.Structure):
    _fields_ = [("batch", C.c_int32), ("hq", C.c_int32), ("hkv", C.c_int32), ("d", C.c_int32),
                ("chunk", C.c_int32), ("n_max", C.c_int32), ("t_max", C.c_int32), ("topk", C.c_int32),
                ("exclude_unselected", C.c_int32), ("scale", C.c_float), ("dtype", C.c_int32),
                ("out_dtype", C.c_int32)]


class gsa_hdesc(C.Structure):
    _fields_ = [("group", C.c_int32), ("topk_meta", C.c_int32), ("m_max", C.c_int32)]


class gsa_h2desc(C.Structure):
    _fields_ = [("level1", gsa_hdesc), ("level2", gsa_hdesc)]


_lib = None


def load(path: Path | None = None) -> C.CDLL:
    """Load libgsa.so (built in-tree by long_context_gsa_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = Path(path) if path else LIB
    if not p.exists():
        raise RuntimeError(f"{p} is missing: build it with `python -m long_context_gsa_b200.build` "
                           "(the GSA kernels have no CPU fallback)")
    lib = C.CDLL(str(p))
    vp, sz, i32 = C.c_void_p, C.c_size_t, C.c_int32
    D, H = C.POINTER(gsa_desc), C.POINTER(gsa_hdesc)
    sig = {
        "gsa_status_string": ([i32], C.c_char_p),
        "gsa_version": ([], i32),
        "gsa_workspace_bytes": ([D, i32, H], sz),
        "gsa_workspace_init": ([vp, sz, vp], i32),
        "gsa_workspace_status": ([vp, sz, vp, C.POINTER(C.c_uint32)], i32),
        "gsa_score_gists": ([D, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "gsa_topk_select": ([D, vp, vp, vp, vp, vp, sz, vp], i32),
        "gsa_topp_select": ([D, vp, vp, C.c_float, vp, vp, vp, vp, sz, vp], i32),
        "gsa_unfold_attend": ([D, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, sz, vp], i32),
        "gsa_decode": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "hgsa_select": ([D, H, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "hgsa_decode": ([D, H, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "hgsa2_select": ([D, C.POINTER(gsa_h2desc)] + [vp] * 13 + [sz, vp], i32),
        "gsa_decode_backward": ([D] + [vp] * 17, i32),
        "gsa_gist_step": ([D] + [vp] * 12 + [sz, vp], i32),
        "gsa_multiquery_select": ([D] + [vp] * 5 + [sz, vp], i32),
        "hgsa2_decode": ([D, C.POINTER(gsa_h2desc)] + [vp] * 18 + [sz, vp], i32),
        "gsa_prefill_score": ([D, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "gsa_prefill_attend": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "gsa_prefill": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32),
        "gsa_decode_noalloc": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], i32),
        "gsa_noalloc_status": ([vp, C.POINTER(C.c_uint32)], i32),
        "gsa_score_select": ([D] + [vp] * 8 + [sz, vp], i32),
    }
    for name, (argt, rest) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = argt
        fn.restype = rest
    if path is None:
        _lib = lib
    return lib


# ------------------------------------------------------------- marshalling
_TORCH_DT = {GSA_F32: torch.float32, GSA_BF16: torch.bfloat16}


def make_desc(batch, hq, hkv, d, chunk, n_max, t_max, topk, exclude_unselected=False, scale=0.0,
              dtype=GSA_BF16, out_dtype=GSA_F32) -> gsa_desc:
    return gsa_desc(batch, hq, hkv, d, chunk, n_max, t_max, topk, int(bool(exclude_unselected)), float(scale),
                    dtype, out_dtype)


def make_hdesc(group, topk_meta, m_max) -> gsa_hdesc:
    return gsa_hdesc(group, topk_meta, m_max)


def make_h2desc(level1: gsa_hdesc, level2: gsa_hdesc) -> gsa_h2desc:
    return gsa_h2desc(level1, level2)


def _n(desc, what, m_max=0, k=None):
    """Element count of one C ABI buffer for `desc` (layouts of include/gsa.h)."""
    B, hq, hkv, d = desc.batch, desc.hq, desc.hkv, desc.d
    k = desc.topk if k is None else k
    return {
        "q": B * hq * d,                        # q, out, d_q, k_new-per-head rows
        "kv_new": B * hkv * d,                  # k_new, v_new
        "gists": B * hkv * desc.n_max * d,      # gist_k, gist_v and their gradients
        "raw": B * hkv * desc.t_max * d,        # raw_k, raw_v and their gradients
        "meta": B * hkv * m_max * d,            # meta_k, meta_v (m_max rows)
        "batch": B,                             # n_gists, own_len
        "heads": B * hq,                        # lse, sel_count
        "scores": B * hq * desc.n_max,
        "sel": B * hq * k,                      # sel_idx, sel_score, meta_idx
        "rows_q": B * hq * desc.t_max * d,      # prefill q_raw / out_raw, multi-query q
        "rows_gq": B * hq * desc.n_max * d,     # prefill q_gist / out_gist
        "rows_sel": B * hq * desc.t_max * k,    # prefill / multi-query selections
    }[what]


def _ptr(t, dtype=None, name="tensor", optional=False, numel=None):
    """Data pointer of `t` after the checks the C ABI relies on: a contiguous
    CUDA tensor of `dtype` holding at least `numel` elements (the size its
    layout in include/gsa.h implies for the descriptor).  A short buffer is
    rejected here, before the library could read or write past its end."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the descriptor needs at least {numel}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the GSA path has no CPU implementation)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _check(fn, st):
    if st != GSA_OK:
        raise GsaError(fn, st, load().gsa_status_string(st).decode())


def _ws(ws):
    if not isinstance(ws, torch.Tensor) or not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous CUDA tensor")
    return C.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def gsa_status_string(status: int) -> str:
    return load().gsa_status_string(status).decode()


def gsa_version() -> int:
    return int(load().gsa_version())


def gsa_workspace_bytes(desc: gsa_desc, op: int = GSA_OP_DECODE, hdesc=None) -> int:
    """hdesc: a gsa_hdesc for GSA_OP_HGSA, a gsa_h2desc for GSA_OP_HGSA2 (its level1 is passed)."""
    if isinstance(hdesc, gsa_h2desc):
        ref = C.cast(C.byref(hdesc), C.POINTER(gsa_hdesc))
    else:
        ref = C.byref(hdesc) if hdesc is not None else None
    return int(load().gsa_workspace_bytes(C.byref(desc), op, ref))


def gsa_workspace_init(ws, stream=None):
    p, n = _ws(ws)
    _check("gsa_workspace_init", load().gsa_workspace_init(p, n, _stream(stream)))


def gsa_workspace_status(ws, stream=None) -> int:
    p, n = _ws(ws)
    flags = C.c_uint32(0)
    st = load().gsa_workspace_status(p, n, _stream(stream), C.byref(flags))
    if st not in (GSA_OK, GSA_ERR_TIMEOUT):
        _check("gsa_workspace_status", st)
    return int(flags.value)


def gsa_score_gists(desc, q, gist_k, gist_v, n_gists, scores, ws, stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("gsa_score_gists", load().gsa_score_gists(
        C.byref(desc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
        _ptr(gist_v, dt, "gist_v", True, _n(desc, "gists")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(scores, torch.float32, "scores", numel=_n(desc, "scores")), *_ws(ws), _stream(stream)))


def gsa_topk_select(desc, scores, n_gists, sel_idx, sel_score, ws, stream=None):
    _check("gsa_topk_select", load().gsa_topk_select(
        C.byref(desc), _ptr(scores, torch.float32, "scores", numel=_n(desc, "scores")),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")), *_ws(ws), _stream(stream)))


def gsa_topp_select(desc, scores, n_gists, top_p, sel_idx, sel_score, sel_count, ws, stream=None):
    _check("gsa_topp_select", load().gsa_topp_select(
        C.byref(desc), _ptr(scores, torch.float32, "scores", numel=_n(desc, "scores")),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch), C.c_float(float(top_p)),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")),
        _ptr(sel_count, torch.int32, "sel_count", True, _n(desc, "heads")), *_ws(ws), _stream(stream)))


def gsa_unfold_attend(desc, q, raw_k, raw_v, gist_v, n_gists, own_len, sel_idx, sel_score, prior, out, lse, ws,
                      stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("gsa_unfold_attend", load().gsa_unfold_attend(
        C.byref(desc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(raw_k, dt, "raw_k", numel=_n(desc, "raw")),
        _ptr(raw_v, dt, "raw_v", numel=_n(desc, "raw")), _ptr(gist_v, dt, "gist_v", True, _n(desc, "gists")),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")), int(prior),
        _ptr(out, _TORCH_DT[desc.out_dtype], "out", numel=_n(desc, "q")),
        _ptr(lse, torch.float32, "lse", True, _n(desc, "heads")), *_ws(ws), _stream(stream)))


def gsa_score_select(desc, q, gist_k, gist_v, n_gists, scores, sel_idx, sel_score, ws, stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("gsa_score_select", load().gsa_score_select(
        C.byref(desc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
        _ptr(gist_v, dt, "gist_v", True, _n(desc, "gists")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(scores, torch.float32, "scores", True, _n(desc, "scores")),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")), *_ws(ws), _stream(stream)))


def _decode_ptrs(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse, sel_idx, sel_score):
    """The pointer arguments shared by gsa_decode and gsa_decode_noalloc."""
    dt = _TORCH_DT[desc.dtype]
    return (_ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
            _ptr(gist_v, dt, "gist_v", numel=_n(desc, "gists")), _ptr(raw_k, dt, "raw_k", numel=_n(desc, "raw")),
            _ptr(raw_v, dt, "raw_v", numel=_n(desc, "raw")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
            _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
            _ptr(out, _TORCH_DT[desc.out_dtype], "out", numel=_n(desc, "q")),
            _ptr(lse, torch.float32, "lse", True, _n(desc, "heads")),
            _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")),
            _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")))


def gsa_decode(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse=None, sel_idx=None,
               sel_score=None, ws=None, stream=None):
    _check("gsa_decode", load().gsa_decode(
        C.byref(desc), *_decode_ptrs(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse, sel_idx,
                                     sel_score), *_ws(ws), _stream(stream)))


def hgsa_select(desc, hdesc, q, meta_k, meta_v, gist_k, gist_v, n_gists, meta_idx, sel_idx, sel_score, ws,
                stream=None):
    dt = _TORCH_DT[desc.dtype]
    nm = _n(desc, "meta", m_max=hdesc.m_max)
    _check("hgsa_select", load().hgsa_select(
        C.byref(desc), C.byref(hdesc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(meta_k, dt, "meta_k", numel=nm),
        _ptr(meta_v, dt, "meta_v", True, nm), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
        _ptr(gist_v, dt, "gist_v", True, _n(desc, "gists")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(meta_idx, torch.int32, "meta_idx", numel=_n(desc, "sel", k=hdesc.topk_meta)),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", numel=_n(desc, "sel")), *_ws(ws), _stream(stream)))


def hgsa_decode(desc, hdesc, q, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse=None,
                meta_idx=None, sel_idx=None, sel_score=None, ws=None, stream=None):
    dt = _TORCH_DT[desc.dtype]
    nm = _n(desc, "meta", m_max=hdesc.m_max)
    _check("hgsa_decode", load().hgsa_decode(
        C.byref(desc), C.byref(hdesc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(meta_k, dt, "meta_k", numel=nm),
        _ptr(meta_v, dt, "meta_v", numel=nm), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
        _ptr(gist_v, dt, "gist_v", numel=_n(desc, "gists")), _ptr(raw_k, dt, "raw_k", numel=_n(desc, "raw")),
        _ptr(raw_v, dt, "raw_v", numel=_n(desc, "raw")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
        _ptr(out, _TORCH_DT[desc.out_dtype], "out", numel=_n(desc, "q")),
        _ptr(lse, torch.float32, "lse", True, _n(desc, "heads")),
        _ptr(meta_idx, torch.int32, "meta_idx", True, _n(desc, "sel", k=hdesc.topk_meta)),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")), *_ws(ws), _stream(stream)))


def _hgsa2_ptrs(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, v_optional):
    dt = _TORCH_DT[desc.dtype]
    n2 = _n(desc, "meta", m_max=h2desc.level2.m_max)
    n1 = _n(desc, "meta", m_max=h2desc.level1.m_max)
    return (_ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(meta2_k, dt, "meta2_k", numel=n2),
            _ptr(meta2_v, dt, "meta2_v", v_optional, n2), _ptr(meta_k, dt, "meta_k", numel=n1),
            _ptr(meta_v, dt, "meta_v", v_optional, n1), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
            _ptr(gist_v, dt, "gist_v", v_optional, _n(desc, "gists")))


def hgsa2_select(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, n_gists, meta2_idx, meta_idx,
                 sel_idx, sel_score, ws, stream=None):
    _check("hgsa2_select", load().hgsa2_select(
        C.byref(desc), C.byref(h2desc),
        *_hgsa2_ptrs(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, True),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(meta2_idx, torch.int32, "meta2_idx", numel=_n(desc, "sel", k=h2desc.level2.topk_meta)),
        _ptr(meta_idx, torch.int32, "meta_idx", numel=_n(desc, "sel", k=h2desc.level1.topk_meta)),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", numel=_n(desc, "sel")), *_ws(ws), _stream(stream)))


def hgsa2_decode(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, raw_k, raw_v, n_gists, own_len,
                 out, lse=None, meta2_idx=None, meta_idx=None, sel_idx=None, sel_score=None, ws=None, stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("hgsa2_decode", load().hgsa2_decode(
        C.byref(desc), C.byref(h2desc),
        *_hgsa2_ptrs(desc, h2desc, q, meta2_k, meta2_v, meta_k, meta_v, gist_k, gist_v, False),
        _ptr(raw_k, dt, "raw_k", numel=_n(desc, "raw")), _ptr(raw_v, dt, "raw_v", numel=_n(desc, "raw")),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
        _ptr(out, _TORCH_DT[desc.out_dtype], "out", numel=_n(desc, "q")),
        _ptr(lse, torch.float32, "lse", True, _n(desc, "heads")),
        _ptr(meta2_idx, torch.int32, "meta2_idx", True, _n(desc, "sel", k=h2desc.level2.topk_meta)),
        _ptr(meta_idx, torch.int32, "meta_idx", True, _n(desc, "sel", k=h2desc.level1.topk_meta)),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "sel")), *_ws(ws), _stream(stream)))


def gsa_multiquery_select(desc, q, gist_k, sel_idx, sel_score, ws, stream=None):
    _check("gsa_multiquery_select", load().gsa_multiquery_select(
        C.byref(desc), _ptr(q, torch.bfloat16, "q", numel=_n(desc, "rows_q")),
        _ptr(gist_k, torch.bfloat16, "gist_k", numel=_n(desc, "gists")),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "rows_sel")),
        _ptr(sel_score, torch.float32, "sel_score", numel=_n(desc, "rows_sel")), *_ws(ws), _stream(stream)))


def gsa_gist_step(desc, q, k_new, v_new, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse, ws, stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("gsa_gist_step", load().gsa_gist_step(
        C.byref(desc), _ptr(q, dt, "q", numel=_n(desc, "q")), _ptr(k_new, dt, "k_new", numel=_n(desc, "kv_new")),
        _ptr(v_new, dt, "v_new", numel=_n(desc, "kv_new")), _ptr(gist_k, dt, "gist_k", numel=_n(desc, "gists")),
        _ptr(gist_v, dt, "gist_v", numel=_n(desc, "gists")), _ptr(raw_k, dt, "raw_k", numel=_n(desc, "raw")),
        _ptr(raw_v, dt, "raw_v", numel=_n(desc, "raw")), _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
        _ptr(out, _TORCH_DT[desc.out_dtype], "out", numel=_n(desc, "q")),
        _ptr(lse, torch.float32, "lse", True, _n(desc, "heads")), *_ws(ws), _stream(stream)))


def gsa_decode_backward(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, sel_idx, out, lse, d_out, d_q,
                        d_gist_k, d_gist_v, d_raw_k, d_raw_v, stream=None):
    dt = _TORCH_DT[desc.dtype]
    f = torch.float32
    nq, ng, nr = _n(desc, "q"), _n(desc, "gists"), _n(desc, "raw")
    _check("gsa_decode_backward", load().gsa_decode_backward(
        C.byref(desc), _ptr(q, dt, "q", numel=nq), _ptr(gist_k, dt, "gist_k", numel=ng),
        _ptr(gist_v, dt, "gist_v", numel=ng), _ptr(raw_k, dt, "raw_k", numel=nr), _ptr(raw_v, dt, "raw_v", numel=nr),
        _ptr(n_gists, torch.int32, "n_gists", numel=desc.batch),
        _ptr(own_len, torch.int32, "own_len", numel=desc.batch),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "sel")), _ptr(out, f, "out", numel=nq),
        _ptr(lse, f, "lse", numel=_n(desc, "heads")), _ptr(d_out, f, "d_out", numel=nq),
        _ptr(d_q, f, "d_q", numel=nq), _ptr(d_gist_k, f, "d_gist_k", numel=ng),
        _ptr(d_gist_v, f, "d_gist_v", numel=ng), _ptr(d_raw_k, f, "d_raw_k", numel=nr),
        _ptr(d_raw_v, f, "d_raw_v", numel=nr), _stream(stream)))


def gsa_prefill_score(desc, q_raw, q_gist, k_gist, sel_idx, sel_score, ws, stream=None):
    dt = _TORCH_DT[desc.dtype]
    _check("gsa_prefill_score", load().gsa_prefill_score(
        C.byref(desc), _ptr(q_raw, dt, "q_raw", numel=_n(desc, "rows_q")),
        _ptr(q_gist, dt, "q_gist", numel=_n(desc, "rows_gq")), _ptr(k_gist, dt, "k_gist", numel=_n(desc, "gists")),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "rows_sel")),
        _ptr(sel_score, torch.float32, "sel_score", numel=_n(desc, "rows_sel")), *_ws(ws), _stream(stream)))


def _prefill_inputs(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist):
    dt = _TORCH_DT[desc.dtype]
    return (_ptr(q_raw, dt, "q_raw", numel=_n(desc, "rows_q")), _ptr(k_raw, dt, "k_raw", numel=_n(desc, "raw")),
            _ptr(v_raw, dt, "v_raw", numel=_n(desc, "raw")), _ptr(q_gist, dt, "q_gist", numel=_n(desc, "rows_gq")),
            _ptr(k_gist, dt, "k_gist", numel=_n(desc, "gists")), _ptr(v_gist, dt, "v_gist", numel=_n(desc, "gists")))


def gsa_prefill_attend(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist, sel_idx, sel_score, out_raw, out_gist, ws,
                       stream=None):
    odt = _TORCH_DT[desc.out_dtype]
    _check("gsa_prefill_attend", load().gsa_prefill_attend(
        C.byref(desc), *_prefill_inputs(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist),
        _ptr(sel_idx, torch.int32, "sel_idx", numel=_n(desc, "rows_sel")),
        _ptr(sel_score, torch.float32, "sel_score", numel=_n(desc, "rows_sel")),
        _ptr(out_raw, odt, "out_raw", numel=_n(desc, "rows_q")),
        _ptr(out_gist, odt, "out_gist", numel=_n(desc, "rows_gq")), *_ws(ws), _stream(stream)))


def gsa_prefill(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist, out_raw, out_gist, sel_idx=None, sel_score=None,
                ws=None, stream=None):
    odt = _TORCH_DT[desc.out_dtype]
    _check("gsa_prefill", load().gsa_prefill(
        C.byref(desc), *_prefill_inputs(desc, q_raw, k_raw, v_raw, q_gist, k_gist, v_gist),
        _ptr(sel_idx, torch.int32, "sel_idx", True, _n(desc, "rows_sel")),
        _ptr(sel_score, torch.float32, "sel_score", True, _n(desc, "rows_sel")),
        _ptr(out_raw, odt, "out_raw", numel=_n(desc, "rows_q")),
        _ptr(out_gist, odt, "out_gist", numel=_n(desc, "rows_gq")), *_ws(ws), _stream(stream)))


def gsa_decode_noalloc(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse=None, sel_idx=None,
                       sel_score=None, stream=None):
    """gsa_decode without a workspace argument (the library's built-in
    scratch array is used; see include/gsa.h for its limit and the rule
    that calls must not overlap on the GPU)."""
    _check("gsa_decode_noalloc", load().gsa_decode_noalloc(
        C.byref(desc), *_decode_ptrs(desc, q, gist_k, gist_v, raw_k, raw_v, n_gists, own_len, out, lse, sel_idx,
                                     sel_score), _stream(stream)))


def gsa_noalloc_status(stream=None) -> int:
    """GSA_DEVERR_* bits left by gsa_decode_noalloc on the current device
    (read and cleared; synchronises the stream)."""
    flags = C.c_uint32(0)
    st = load().gsa_noalloc_status(_stream(stream), C.byref(flags))
    if st not in (GSA_OK, GSA_ERR_TIMEOUT):
        _check("gsa_noalloc_status", st)
    return int(flags.value)
