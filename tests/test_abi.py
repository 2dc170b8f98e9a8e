"""The C ABI: the library loads, exports every function ``include/kda.h``
declares, and rejects bad arguments on the host before touching a device.

None of these calls launches a kernel: each returns from the host-side
argument checks (or is a query), so the file runs without a GPU.
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_116_b200 as kda
from gated_delta_rule_116_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kda_chunk_fwd", "kda_recurrent_step", "kda_workspace_bytes", "kda_strerror"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in kda.h but not exported"


def test_every_exported_entry_point_is_declared():
    """The library's exported C entry points (``kda_*``, from its dynamic symbol
    table) are exactly those the header documents; debug counters exist only in
    debug builds."""
    import subprocess
    nm = subprocess.run(["nm", "-D", "--defined-only", kda.LIB_PATH], capture_output=True, text=True)
    if nm.returncode != 0:
        pytest.skip("nm is not available")
    exported = {line.split()[-1] for line in nm.stdout.splitlines()
                if line.split() and line.split()[-1].startswith("kda_")}
    exported = {n for n in exported if not n.startswith("kda_debug_")}
    assert exported == set(declared_functions())


def test_status_names(lib):
    expect = {0: "KDA_OK", -1: "KDA_ERR_INVALID_ARG", -2: "KDA_ERR_UNSUPPORTED",
              -3: "KDA_ERR_ALIGNMENT", -4: "KDA_ERR_WORKSPACE", -5: "KDA_ERR_CUDA",
              -6: "KDA_ERR_DEVICE_TIMEOUT"}
    for code, name in expect.items():
        assert lib.kda_strerror(code).decode() == name
    assert lib.kda_version() >= 10000


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


def chunk(lib, engine=0, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, out=FAKE, ST=None,
          B=1, T=64, H=2, dk=128, dv=128, C=64, dtype=0, ws=None, wsb=0):
    return lib.kda_chunk_fwd_engine(engine, q, k, v, la, beta, S0, out, ST, B, T, H, dk, dv, C,
                                    dtype, ws, wsb, None)


def detail(lib):
    return lib.kda_last_error_detail().decode()


@pytest.mark.parametrize("field", ["q", "k", "v", "la", "beta", "out"])
def test_chunk_null_pointer(lib, field):
    assert chunk(lib, **{field: None}) == -1
    assert detail(lib)


@pytest.mark.parametrize("field", ["q", "v", "la", "out", "S0", "ST"])
def test_chunk_misaligned_pointer(lib, field):
    assert chunk(lib, **{field: FAKE + 2}) == -3
    assert "aligned" in detail(lib)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=5), -1), (dict(B=-1), -1), (dict(T=-3), -1), (dict(dk=0), -1),
    (dict(dk=256), -2), (dict(dv=130), -2), (dict(dv=6), -2), (dict(C=48), -2),
    (dict(C=128), -2), (dict(engine=9), -1), (dict(engine=3, C=16), -2), (dict(engine=3, dtype=1), -2),
    (dict(engine=2), -1), (dict(engine=3, dk=64), -2), (dict(engine=3, C=32), -2),
    (dict(B=2, T=2**30), -2), (dict(B=2**15, H=2**15), -2), (dict(engine=1, B=3, T=2**30), -2),
])
def test_chunk_rejects(lib, kw, code):
    assert chunk(lib, **kw) == code
    assert detail(lib)


@pytest.mark.parametrize("engine", [0, 3])
def test_chunk_workspace_missing_or_short(lib, engine):
    """The cluster engine (also what engine 0 picks for this shape) needs a workspace of
    kda_workspace_bytes(); without one, or with fewer bytes, the call fails on the
    host with KDA_ERR_WORKSPACE before any launch."""
    need = lib.kda_workspace_bytes(1, 64, 2, 128, 128, 64, 0)
    assert need > 0
    assert chunk(lib, engine=engine) == -4
    assert "workspace" in detail(lib)
    assert chunk(lib, engine=engine, ws=FAKE, wsb=need - 16) == -4


def test_chunk_empty_batch_is_noop(lib):
    assert chunk(lib, B=0, q=None, k=None, v=None, la=None, beta=None, out=None) == 0
    assert chunk(lib, H=0, q=None, k=None, v=None, la=None, beta=None, out=None) == 0


def step(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, state=FAKE, slot=None, out=FAKE,
         N=4, H=2, dk=128, dv=128, dtype=0):
    return lib.kda_recurrent_step(q, k, v, la, beta, state, slot, out, N, H, dk, dv, dtype, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "la", "beta", "state", "out"])
def test_step_null_pointer(lib, field):
    assert step(lib, **{field: None}) == -1


@pytest.mark.parametrize("kw,code", [
    (dict(state=FAKE + 4), -3), (dict(slot=FAKE + 8), -3), (dict(dtype=2), -1), (dict(N=-1), -1),
    (dict(dk=129), -2), (dict(dv=10), -2), (dict(N=2**16, H=2**14), -2),
])
def test_step_rejects(lib, kw, code):
    assert step(lib, **kw) == code


def test_step_empty_is_noop(lib):
    assert step(lib, N=0, q=None, k=None, v=None, la=None, beta=None, state=None, out=None) == 0


def test_workspace_query(lib):
    for args in [(1, 64, 2, 16, 16, 16, 1), (8, 4096, 32, 128, 128, 64, 0), (0, 10, 1, 128, 128, 64, 0)]:
        assert lib.kda_workspace_bytes(*args) >= 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError, match="CUDA"):
        kda.chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1), chunk=16)


def bwd(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, go=FAKE, gST=None, gq=FAKE,
        gk=FAKE, gv=FAKE, gla=FAKE, gb=FAKE, gS0=None, B=1, T=32, H=2, dk=128, dv=128, dtype=0,
        ws=None, wsb=0):
    return lib.kda_chunk_bwd(q, k, v, la, beta, S0, go, gST, gq, gk, gv, gla, gb, gS0, B, T, H, dk,
                             dv, dtype, ws, wsb, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "la", "beta", "go", "gq", "gk", "gv", "gla", "gb"])
def test_bwd_null_pointer(lib, field):
    assert bwd(lib, **{field: None}) == -1
    assert detail(lib)


@pytest.mark.parametrize("kw,code", [
    (dict(gq=FAKE + 4), -3), (dict(gS0=FAKE + 8), -3), (dict(dtype=3), -1), (dict(B=-1), -1),
    (dict(dk=0), -1), (dict(dk=129), -2), (dict(dv=200), -2), (dict(B=2, T=2**30), -2),
])
def test_bwd_rejects(lib, kw, code):
    assert bwd(lib, **kw) == code
    assert detail(lib)


def test_bwd_workspace_missing_or_short(lib):
    need = lib.kda_bwd_workspace_bytes(1, 32, 2, 128, 128, 0)
    # two 16-token chunks of 128 x 128 fp32 entry states per head, plus fp32 dq and dk
    assert need == (2 * 2 * 128 * 128 + 2 * 32 * 2 * 128) * 4
    assert bwd(lib) == -4 and "workspace" in detail(lib)
    assert bwd(lib, ws=FAKE, wsb=need - 16) == -4


def test_bwd_empty_batch_is_noop(lib):
    none = dict(q=None, k=None, v=None, la=None, beta=None, go=None, gq=None, gk=None, gv=None,
                gla=None, gb=None)
    assert bwd(lib, B=0, **none) == 0
    assert bwd(lib, H=0, **none) == 0
    assert lib.kda_bwd_workspace_bytes(0, 32, 2, 128, 128, 0) == 0


def test_binding_backward_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 16)
    la = torch.zeros(1, 4, 1, 16)
    b = torch.zeros(1, 4, 1)
    with pytest.raises(ValueError, match="CUDA"):
        kda.chunk_bwd(x, x, x, la, b, x)


def varlen(lib, q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, cu=FAKE, slot=None, S0=None, out=FAKE,
           ST=None, N=2, TT=64, H=2, dk=128, dv=128, dtype=0):
    return lib.kda_chunk_fwd_varlen(q, k, v, la, beta, cu, slot, S0, out, ST, N, TT, H, dk, dv, dtype,
                                    None)


@pytest.mark.parametrize("kw,code", [
    (dict(cu=None), -1), (dict(cu=FAKE + 2), -3), (dict(slot=FAKE + 2), -3), (dict(q=None), -1),
    (dict(out=FAKE + 8), -3),
    (dict(dtype=2), -1), (dict(N=-1), -1), (dict(TT=-1), -1), (dict(dk=0), -1), (dict(dv=129), -2),
    (dict(N=2**15, H=2**15), -2),
])
def test_varlen_rejects(lib, kw, code):
    assert varlen(lib, **kw) == code
    assert detail(lib)


def test_varlen_empty_is_noop(lib):
    assert varlen(lib, N=0, cu=None, q=None, k=None, v=None, la=None, beta=None, out=None) == 0
    assert varlen(lib, H=0, cu=None, q=None, k=None, v=None, la=None, beta=None, out=None) == 0
