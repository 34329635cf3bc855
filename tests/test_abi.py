"""libgsa.so builds for sm_100a, loads, exports every entry point declared in
include/gsa.h, and rejects bad arguments on the host before any CUDA call.
CPU only: no kernel is launched here."""
import ctypes as C
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    from long_context_gsa_b200 import build, load
    build.build_library()
    return load()


def declared_functions():
    text = (ROOT / "include" / "gsa.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/gsa.h but not exported"
    from long_context_gsa_b200 import EXPORTS
    assert set(EXPORTS) == set(names)


def test_status_strings_and_version(lib):
    from long_context_gsa_b200 import gsa_status_string, gsa_version
    assert gsa_status_string(0) == "GSA_OK"
    assert "workspace" in gsa_status_string(3)
    assert gsa_version() >= 100


def _desc(**kw):
    """Raw descriptor (no normalisation, so invalid field values reach the C checks)."""
    from long_context_gsa_b200 import gsa_desc
    base = dict(batch=2, hq=8, hkv=2, d=128, chunk=16, n_max=64, t_max=64 * 16 + 16, topk=8, exclude_unselected=0,
                scale=0.0, dtype=1, out_dtype=0)
    base.update(kw)
    return gsa_desc(*[base[f] for f, _ in gsa_desc._fields_])


def test_workspace_bytes(lib):
    from long_context_gsa_b200 import GSA_OP_DECODE, GSA_OP_HGSA, GSA_OP_PREFILL, gsa_workspace_bytes, make_hdesc
    d = _desc()
    n = gsa_workspace_bytes(d, GSA_OP_DECODE)
    assert n > 2 * 8 * 64 * 4 and n % 256 == 0
    assert gsa_workspace_bytes(_desc(d=96), GSA_OP_DECODE) == 0
    assert gsa_workspace_bytes(_desc(hq=6, hkv=4), GSA_OP_DECODE) == 0
    h = make_hdesc(4, 4, 16)
    assert gsa_workspace_bytes(d, GSA_OP_HGSA, h) > n
    assert gsa_workspace_bytes(d, GSA_OP_HGSA, None) == 0
    assert gsa_workspace_bytes(_desc(n_max=8, t_max=128, topk=4), GSA_OP_PREFILL) > 0


# Fake device addresses are only ever passed to calls that must reject them
# during host-side validation, before anything is enqueued.  Should a check
# ever let one through, the call would enqueue work on a bogus address, so
# these tests never run where a GPU is visible.
A = 1 << 20  # aligned, never dereferenced


def _no_gpu():
    import torch
    return not torch.cuda.is_available()


cpu_only = pytest.mark.skipif(not _no_gpu(), reason="fake-pointer validation tests run only without a GPU")


@cpu_only
@pytest.mark.parametrize("bad,code", [
    (dict(d=96), 2), (dict(hq=6, hkv=4), 1), (dict(chunk=0), 2), (dict(topk=-1), 1), (dict(topk=5000), 2),
    (dict(exclude_unselected=2), 1), (dict(dtype=7), 1), (dict(batch=0), 1), (dict(hq=64, hkv=2), 2),
])
def test_bad_descriptor_rejected(lib, bad, code):
    d = _desc(**bad)
    st = lib.gsa_decode(C.byref(d), A, A, A, A, A, A, A, A, None, None, None, A, 1 << 40, None)
    assert st == code


@cpu_only
def test_null_and_misaligned_pointers_rejected(lib):
    d = _desc()
    assert lib.gsa_decode(C.byref(d), None, A, A, A, A, A, A, A, None, None, None, A, 1 << 40, None) == 1
    assert lib.gsa_decode(C.byref(d), A + 4, A, A, A, A, A, A, A, None, None, None, A, 1 << 40, None) == 1
    assert lib.gsa_score_gists(C.byref(d), A, A, None, A, A, A, 1 << 40, None) == 1  # gist_v needed by default
    assert lib.gsa_unfold_attend(C.byref(d), A, A, A, None, A, A, A, None, 0, A, None, A, 1 << 40, None) == 1


@cpu_only
def test_small_workspace_rejected(lib):
    d = _desc()
    assert lib.gsa_decode(C.byref(d), A, A, A, A, A, A, A, A, None, None, None, A, 1024, None) == 3
    assert lib.gsa_topk_select(C.byref(d), A, A, A, None, A, 16, None) == 3


def test_binding_refuses_cpu_tensors(lib):
    import torch
    from long_context_gsa_b200 import gsa_decode
    d = _desc()
    t = torch.zeros(4)
    with pytest.raises((ValueError, TypeError)):
        gsa_decode(d, t, t, t, t, t, t, t, t, ws=t)


def test_workspace_bytes_new_ops(lib):
    from long_context_gsa_b200 import GSA_OP_DECODE, GSA_OP_GIST_STEP, GSA_OP_MULTIQUERY, gsa_workspace_bytes
    d = _desc()
    assert gsa_workspace_bytes(d, GSA_OP_GIST_STEP) > 0
    # the gist step ignores topk: its workspace does not grow with it
    assert gsa_workspace_bytes(_desc(topk=512), GSA_OP_GIST_STEP) == gsa_workspace_bytes(_desc(topk=0), GSA_OP_GIST_STEP)
    mq = _desc(topk=16, t_max=300)
    assert gsa_workspace_bytes(mq, GSA_OP_MULTIQUERY) > 2 * 8 * 300 * 4
    assert gsa_workspace_bytes(_desc(topk=16, dtype=0), GSA_OP_MULTIQUERY) == 0  # fp32 inputs: not built
    assert gsa_workspace_bytes(_desc(topk=65), GSA_OP_MULTIQUERY) == 0
    assert gsa_workspace_bytes(_desc(topk=0), GSA_OP_MULTIQUERY) == 0
    assert gsa_workspace_bytes(d, 99) == 0
    assert gsa_workspace_bytes(d, GSA_OP_DECODE) > 0


@cpu_only
def test_new_entry_points_reject_bad_arguments(lib):
    d = _desc()
    f = C.c_float
    # top-p: NaN threshold, k beyond 256
    assert lib.gsa_topp_select(C.byref(d), A, A, f(float("nan")), A, A, A, A, 1 << 40, None) == 1
    assert lib.gsa_topp_select(C.byref(_desc(topk=300)), A, A, f(0.5), A, A, A, A, 1 << 40, None) == 2
    # backward: a missing gradient buffer, a misaligned one, a bad descriptor
    args = [A] * 16
    bad = list(args)
    bad[13] = None  # d_gist_k
    assert lib.gsa_decode_backward(C.byref(d), *bad, None) == 1
    bad = list(args)
    bad[12] = A + 4  # d_q
    assert lib.gsa_decode_backward(C.byref(d), *bad, None) == 1
    assert lib.gsa_decode_backward(C.byref(_desc(d=96)), *args, None) == 2
    # gist step: a missing count array, a workspace too small
    assert lib.gsa_gist_step(C.byref(d), A, A, A, A, A, A, A, None, A, A, None, A, 1 << 40, None) == 1
    assert lib.gsa_gist_step(C.byref(d), A, A, A, A, A, A, A, A, A, A, None, A, 256, None) == 3
    # multi-query: unsupported head size / k, missing output, small workspace
    mq = _desc(topk=16, t_max=300)
    assert lib.gsa_multiquery_select(C.byref(_desc(d=96, topk=16)), A, A, A, A, A, 1 << 40, None) == 2
    assert lib.gsa_multiquery_select(C.byref(_desc(dtype=0, topk=16)), A, A, A, A, A, 1 << 40, None) == 2  # fp32
    assert lib.gsa_multiquery_select(C.byref(_desc(topk=65)), A, A, A, A, A, 1 << 40, None) == 2
    assert lib.gsa_multiquery_select(C.byref(mq), A, A, None, A, A, 1 << 40, None) == 1
    assert lib.gsa_multiquery_select(C.byref(mq), A, A, A, A, A, 1024, None) == 3


def test_missing_library_fails_loudly(tmp_path):
    """The binding has no fallback: a missing libgsa.so is an error naming the build step."""
    from long_context_gsa_b200 import _abi
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _abi.load(tmp_path / "libgsa.so")


def test_product_path_does_not_import_the_oracle():
    """Only tests, smoke() and the benchmark's CPU leg may touch oracle/: the
    package's sources never import it."""
    pkg = ROOT / "long_context_gsa_b200"
    for f in list(pkg.glob("*.py")) + list((pkg / "csrc").glob("*")):
        text = f.read_text(errors="ignore")
        assert "import oracle" not in text and "from oracle" not in text and "gsa_oracle" not in text, f


def test_binding_sizes_follow_the_header_layouts():
    """The element counts the binding requires are the layouts of include/gsa.h."""
    from long_context_gsa_b200._abi import _n
    d = _desc(batch=3, hq=8, hkv=2, d=64, n_max=50, t_max=816, topk=7)
    assert _n(d, "q") == 3 * 8 * 64
    assert _n(d, "gists") == 3 * 2 * 50 * 64
    assert _n(d, "raw") == 3 * 2 * 816 * 64
    assert _n(d, "meta", m_max=5) == 3 * 2 * 5 * 64
    assert _n(d, "scores") == 3 * 8 * 50
    assert _n(d, "sel") == 3 * 8 * 7 and _n(d, "sel", k=4) == 3 * 8 * 4
    assert _n(d, "heads") == 24 and _n(d, "batch") == 3 and _n(d, "kv_new") == 3 * 2 * 64
    assert _n(d, "rows_q") == 3 * 8 * 816 * 64 and _n(d, "rows_gq") == 3 * 8 * 50 * 64
    assert _n(d, "rows_sel") == 3 * 8 * 816 * 7


def test_binding_rejects_short_buffers_before_any_call(lib):
    """A buffer shorter than its layout needs is refused by the binding (the
    library would otherwise read or write past its end); a longer one is
    accepted by the size check."""
    import torch
    from long_context_gsa_b200 import _abi
    d = _desc(batch=2, hq=4, hkv=2, d=64, n_max=16, t_max=16 * 8 + 8, topk=4)
    short = torch.zeros(2 * 4 * 64 - 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="holds 511 elements"):
        _abi._ptr(short, torch.bfloat16, "q", numel=_abi._n(d, "q"))
    long_ = torch.zeros(2 * 4 * 64 + 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):  # size passes; the device check comes next
        _abi._ptr(long_, torch.bfloat16, "q", numel=_abi._n(d, "q"))
    t = torch.zeros(4)
    # the first pointer of each entry point is checked first, before the workspace
    calls = [
        lambda: _abi.gsa_decode(d, short, t, t, t, t, t, t, t, ws=t),
        lambda: _abi.gsa_decode_noalloc(d, short, t, t, t, t, t, t, t),
        lambda: _abi.gsa_score_gists(d, short, t, t, t, t, t),
        lambda: _abi.gsa_unfold_attend(d, short, t, t, t, t, t, t, t, 1, t, None, t),
        lambda: _abi.gsa_topk_select(d, torch.zeros(2 * 4 * 16 - 1), t, t, None, t),
        lambda: _abi.gsa_gist_step(d, short, t, t, t, t, t, t, t, t, t, None, t),
        lambda: _abi.gsa_decode_backward(d, short, *([t] * 16)),
        lambda: _abi.hgsa_select(d, _abi.make_hdesc(4, 2, 4), short, t, t, t, t, t, t, t, t, t),
        lambda: _abi.gsa_prefill_score(d, short, t, t, t, t, t),
        lambda: _abi.gsa_prefill(d, short, t, t, t, t, t, t, t, ws=t),
        lambda: _abi.gsa_multiquery_select(d, short, t, t, t, t),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError, match="holds"):
            call()


def test_binding_arities_match_the_header(lib):
    """Every ctypes signature has as many arguments as its declaration in
    include/gsa.h."""
    text = re.sub(r"/\*.*?\*/", "", (ROOT / "include" / "gsa.h").read_text(), flags=re.S)
    decls = dict(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(([^)]*)\)\s*;", text, flags=re.M))
    assert len(decls) >= 20, sorted(decls)
    for name, params in decls.items():
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(lib, name).argtypes) == n, f"{name}: binding has {len(getattr(lib, name).argtypes)}, header {n}"
