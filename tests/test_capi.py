"""The C ABI on the host: the library loads without a GPU, exports every
symbol the header declares, and rejects invalid arguments before any launch
(no compute call is made here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pkm.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_key_value_b200 import build
    build.build()
    from sparse_key_value_b200 import _lib
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PKM_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("pkm_forward", "pkm_backward", "embbag_forward", "embbag_backward",
              "pkm_forward_workspace_size", "pkm_backward_workspace_size",
              "embbag_backward_workspace_size", "pkm_get_device_error", "pkm_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} not exported"
    from sparse_key_value_b200 import _lib
    assert set(_lib.EXPORTS) <= set(declared_symbols())


def test_only_the_c_abi_is_exported():
    from sparse_key_value_b200 import _lib
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(declared_symbols())


def test_status_strings(lib):
    for code in range(7):
        assert lib.pkm_status_string(code)
    assert lib.pkm_version() >= 100


def _fwd(**kw):
    from sparse_key_value_b200 import fwd_args
    base = dict(T=64, H=2, d_half=64, n_sub=32, k=8, d_v=64)
    base.update(kw)
    fake = ctypes.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced on the host
    a = fwd_args(**base, query=fake, subkeys=fake, values=fake, out=fake, idx=fake,
                 weights=fake, workspace=fake)
    return a


@pytest.mark.parametrize("bad", [dict(k=0), dict(k=33, n_sub=32), dict(k=65, n_sub=100),
                                 dict(d_half=60), dict(d_v=12), dict(H=0), dict(n_sub=0),
                                 dict(n_sub=46341), dict(T=-1), dict(dtype=7)])
def test_forward_rejects_bad_sizes(lib, bad):
    a = _fwd(**bad)
    a.workspace_bytes = 1 << 40
    assert lib.pkm_forward(ctypes.byref(a), None) == 1


def test_forward_rejects_null_and_misaligned(lib):
    a = _fwd()
    a.workspace_bytes = 1 << 40
    a.query = None
    assert lib.pkm_forward(ctypes.byref(a), None) == 1
    a = _fwd()
    a.workspace_bytes = 1 << 40
    a.values = ctypes.c_void_p((1 << 20) + 8)
    assert lib.pkm_forward(ctypes.byref(a), None) == 1


def test_forward_workspace_checks(lib):
    a = _fwd()
    need = lib.pkm_forward_workspace_size(ctypes.byref(a))
    assert need > 0
    a.workspace_bytes = need - 1
    assert lib.pkm_forward(ctypes.byref(a), None) == 6
    bigger = _fwd(T=128)
    assert lib.pkm_forward_workspace_size(ctypes.byref(bigger)) > need


def test_forward_empty_batch_is_ok_without_gpu(lib):
    a = _fwd(T=0)
    assert lib.pkm_forward(ctypes.byref(a), None) == 0


def test_memplus_requires_all_three_and_bf16(lib):
    a = _fwd(d_model=64)
    a.workspace_bytes = 1 << 40
    a.x = ctypes.c_void_p(1 << 20)
    assert lib.pkm_forward(ctypes.byref(a), None) == 1  # W1, W2 missing
    a.W1 = a.W2 = ctypes.c_void_p(1 << 20)
    a.dtype = 0  # fp32 Memory+
    assert lib.pkm_forward(ctypes.byref(a), None) == 2


def test_embbag_rejects_bad_args(lib):
    P = ctypes.c_void_p
    f = P(1 << 20)
    assert lib.embbag_forward(f, 10, 12, 1, f, f, 4, 3, None, f, None) == 1   # d % 8
    assert lib.embbag_forward(f, 10, 16, 1, f, f, 4, 0, None, f, None) == 1   # B = 0
    assert lib.embbag_forward(None, 10, 16, 1, f, f, 4, 3, None, f, None) == 1
    assert lib.embbag_forward(f, 10, 16, 1, f, f, 0, 3, None, f, None) == 0   # no bags


def test_y_out_requires_memplus_and_alignment(lib):
    a = _fwd()
    a.workspace_bytes = 1 << 40
    a.y_out = ctypes.c_void_p(1 << 20)
    assert lib.pkm_forward(ctypes.byref(a), None) == 1  # plain lookup: no gate, no y_out


def _mp(**kw):
    from sparse_key_value_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)
    base = dict(T=64, d_model=64, d_v=32)
    base.update(kw)
    return _lib.MemplusBwdArgs(base["T"], base["d_model"], base["d_v"], fake, fake, fake, fake,
                               fake, fake, fake, fake, fake, fake, 1 << 40)


def test_memplus_backward_validation(lib):
    assert lib.pkm_memplus_backward(ctypes.byref(_mp(d_model=60)), None) == 1
    assert lib.pkm_memplus_backward(ctypes.byref(_mp(d_v=0)), None) == 1
    a = _mp()
    a.dout = None
    assert lib.pkm_memplus_backward(ctypes.byref(a), None) == 1
    a = _mp()
    a.dW1 = ctypes.c_void_p((1 << 20) + 4)
    assert lib.pkm_memplus_backward(ctypes.byref(a), None) == 1
    a = _mp()
    need = lib.pkm_memplus_backward_workspace_size(ctypes.byref(a))
    a.workspace_bytes = need - 1
    assert lib.pkm_memplus_backward(ctypes.byref(a), None) == 6


def test_qproj_validation(lib):
    from sparse_key_value_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)
    a = _lib.QprojArgs(64, 64, 12, fake, fake, fake, fake, fake, fake, fake, 1 << 40)
    assert lib.pkm_qproj_forward(ctypes.byref(a), None) == 1  # d_q % 8 != 0
    a = _lib.QprojArgs(64, 64, 16, fake, fake, None, fake, fake, fake, fake, 1 << 40)
    assert lib.pkm_qproj_forward(ctypes.byref(a), None) == 1  # no q
    a = _lib.QprojArgs(64, 64, 16, fake, fake, fake, None, fake, fake, fake, 1 << 40)
    assert lib.pkm_qproj_backward(ctypes.byref(a), None) == 1  # no dq
    a = _lib.QprojArgs(64, 64, 16, fake, fake, fake, fake, fake, fake, fake, 16)
    assert lib.pkm_qproj_forward(ctypes.byref(a), None) == 6


def test_sparse_optimizer_validation(lib):
    from sparse_key_value_b200 import _lib
    fake = ctypes.c_void_p(1 << 20)

    def args(**kw):
        base = dict(kind=0, lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8, step=1, n_rows=100, d=64,
                    dtype=1, cap=10)
        base.update(kw)
        return _lib.SparseOptArgs(base["kind"], base["lr"], base["beta1"], base["beta2"],
                                  base["eps"], base["step"], base["n_rows"], base["d"],
                                  base["dtype"], fake, fake, fake, fake, base["cap"], fake, fake)

    assert lib.pkm_sparse_optimizer_step(ctypes.byref(args(d=60)), None) == 1
    assert lib.pkm_sparse_optimizer_step(ctypes.byref(args(kind=2)), None) == 1
    assert lib.pkm_sparse_optimizer_step(ctypes.byref(args(kind=1, beta1=1.0)), None) == 1
    assert lib.pkm_sparse_optimizer_step(ctypes.byref(args(kind=1, step=0)), None) == 1
    assert lib.pkm_sparse_optimizer_step(ctypes.byref(args(lr=float("nan"))), None) == 1
    a = args(kind=1)
    a.m = None
    assert lib.pkm_sparse_optimizer_step(ctypes.byref(a), None) == 1


def _engram(**kw):
    from sparse_key_value_b200 import _lib
    orders = (ctypes.c_int32 * 2)(2, 3)
    seeds = (ctypes.c_uint64 * 4)(1, 2, 3, 4)
    M = (ctypes.c_int64 * 4)(7, 11, 13, 17)
    fake = ctypes.c_void_p(1 << 20)
    base = dict(n_seq=2, L=8, n_orders=2, K=2, orders=ctypes.cast(orders, ctypes.c_void_p),
                seeds=ctypes.cast(seeds, ctypes.c_void_p), rows_per_head=ctypes.cast(M, ctypes.c_void_p),
                d=64, dtype=1, tokens=fake, table=fake, h=fake, v=fake, alpha=None, rows=None,
                e=None)
    base.update(kw)
    a = _lib.EngramArgs(**base)
    a._keep = (orders, seeds, M)
    return a


@pytest.mark.parametrize("bad", [dict(n_orders=0), dict(n_orders=9), dict(K=0), dict(K=65),
                                 dict(L=0), dict(n_seq=-1), dict(d=12), dict(d=8200),
                                 dict(dtype=5), dict(orders=None), dict(seeds=None),
                                 dict(rows_per_head=None), dict(table=None), dict(h=None),
                                 dict(v=None), dict(tokens=ctypes.c_void_p((1 << 20) + 2)),
                                 dict(table=ctypes.c_void_p((1 << 20) + 8)),
                                 dict(alpha=ctypes.c_void_p((1 << 20) + 2))])
def test_engram_rejects_bad_args(lib, bad):
    a = _engram(**bad)
    assert lib.pkm_engram_forward(ctypes.byref(a), None) == 1


def test_engram_rejects_bad_head_config(lib):
    orders = (ctypes.c_int32 * 2)(2, 9)  # order 9 > 8
    a = _engram(orders=ctypes.cast(orders, ctypes.c_void_p))
    assert lib.pkm_engram_forward(ctypes.byref(a), None) == 1
    M = (ctypes.c_int64 * 4)(7, 0, 13, 17)  # an empty head table
    a = _engram(rows_per_head=ctypes.cast(M, ctypes.c_void_p))
    assert lib.pkm_engram_forward(ctypes.byref(a), None) == 1
    M = (ctypes.c_int64 * 4)(1 << 30, 1 << 30, 13, 17)  # 2^31 rows in total
    a = _engram(rows_per_head=ctypes.cast(M, ctypes.c_void_p))
    assert lib.pkm_engram_forward(ctypes.byref(a), None) == 1


def test_engram_empty_batch_is_ok_without_gpu(lib):
    a = _engram(n_seq=0)
    assert lib.pkm_engram_forward(ctypes.byref(a), None) == 0


def test_select_validation(lib):
    bad = _fwd(k=0)
    bad.workspace_bytes = 1 << 40
    assert lib.pkm_select(ctypes.byref(bad), None) == 1
    nq = _fwd()
    nq.query = None
    nq.workspace_bytes = 1 << 40
    assert lib.pkm_select(ctypes.byref(nq), None) == 1
    small = _fwd()
    small.workspace_bytes = 16
    assert lib.pkm_select(ctypes.byref(small), None) == 6
    empty = _fwd(T=0)
    assert lib.pkm_select(ctypes.byref(empty), None) == 0


def test_embbag_range_validation(lib):
    f = ctypes.c_void_p(1 << 20)
    ok = dict(table=f, row_lo=0, n_local=10, d=16, dtype=1, idx=f, w=f, n_bags=0, B=4, out=f)
    call = lambda **kw: lib.embbag_forward_range(*{**ok, **kw}.values(), None)  # noqa: E731
    assert call() == 0                       # empty batch, no launch
    assert call(n_bags=1, row_lo=-1) == 1
    assert call(n_bags=1, n_local=0) == 1
    assert call(n_bags=1, d=12) == 1
    assert call(n_bags=1, B=0) == 1
    assert call(n_bags=1, table=None) == 1
    assert call(n_bags=1, out=ctypes.c_void_p((1 << 20) + 4)) == 1


def test_wait_timeout_check_validation(lib):
    f = ctypes.c_void_p(1 << 20)
    assert lib.pkm_check_wait_timeout(0, f, None) == 1
    assert lib.pkm_check_wait_timeout((1 << 20) + 1, f, None) == 1
    assert lib.pkm_check_wait_timeout(16, None, None) == 1
    assert lib.pkm_check_wait_timeout(16, ctypes.c_void_p((1 << 20) + 2), None) == 1


def test_plain_c_consumer(lib, tmp_path):
    """tests/c_abi_check.c: include/pkm.h compiles as strict C99, a C program
    links libpkm.so and the host-side paths behave as the header says."""
    import shutil
    import subprocess

    from sparse_key_value_b200 import _lib

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
           os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe,
           _lib.LIB_PATH, f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr
