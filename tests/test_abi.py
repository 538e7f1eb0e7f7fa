"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_attention_sum_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(dsa.lib_path()):
        from sparse_attention_sum_b200 import build
        build.build()
    return dsa.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dsa_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(lib, n) is not None


def test_binding_covers_the_header():
    assert set(_declared()) <= set(dsa._SIGS)


def test_status_strings(lib):
    for code, name in dsa.STATUS.items():
        assert lib.dsa_status_string(code).decode() == name
    assert b"sm_100a" in lib.dsa_version()


def test_workspace_size(lib):
    d = dsa.Dims(batch=2, n_q=3, n_kv=100, top_k=8)
    n = dsa.workspace_size(d, dsa.OP_LAYER_FORWARD)
    assert n == ((2 * 3 * 100 * 4 + 255) // 256) * 256 + ((2 * 3 * 8 * 4 + 255) // 256) * 256
    assert dsa.workspace_size(d, dsa.OP_TOPK) == 0
    assert dsa.workspace_size(d, 99) == 0
    assert dsa.workspace_size(dsa.Dims(batch=0, n_q=1, n_kv=1, top_k=1), dsa.OP_LAYER_FORWARD) == 0


def _call(fn, *args):
    st = fn(*args)
    return st, dsa.lib().dsa_last_error().decode()


def test_host_validation_rejects_bad_arguments(lib):
    nul = None
    d = dsa.Dims(batch=1, n_q=4, n_kv=8, idx_heads=2, idx_dim=16, top_k=4, heads=2, kv_heads=1,
                 kd=16, vd=8, kpool=0, out_width=4, dtype=dsa.BF16)
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    st, msg = _call(lib.dsa_index_scores, None, p, p, p, 1.0, p, p, p, p, nul)
    assert st == 1 and "dims" in msg
    st, msg = _call(lib.dsa_index_scores, ctypes.byref(d), nul, p, p, 1.0, p, p, p, p, nul)
    assert st == 1 and "non-NULL" in msg
    st, msg = _call(lib.dsa_topk, ctypes.byref(d), p, p, p, p, 0, p, nul, nul, 0, nul)
    assert st == 1 and "k must be" in msg
    st, msg = _call(lib.dsa_topk, ctypes.byref(d), p, p, p, p, 5000, p, nul, nul, 0, nul)
    assert st == 1
    bad = dsa.Dims(**{**d.as_dict(), "heads": 3, "kv_heads": 2})
    st, msg = _call(lib.dsa_sparse_attend, ctypes.byref(bad), p, p, 16, p, 16, p, 4, 1.0, p, nul, nul)
    assert st == 1 and "divide" in msg
    st, msg = _call(lib.dsa_sparse_attend, ctypes.byref(d), p, p, 8, p, 16, p, 4, 1.0, p, nul, nul)
    assert st == 1 and "k_row_stride" in msg
    bad = dsa.Dims(**{**d.as_dict(), "dtype": 7})
    st, msg = _call(lib.dsa_sparse_attend, ctypes.byref(bad), p, p, 16, p, 16, p, 4, 1.0, p, nul, nul)
    assert st == 1 and "dtype" in msg
    # layer forward: workspace too small is reported as DSA_ERR_WORKSPACE
    st, msg = _call(lib.dsa_layer_forward, ctypes.byref(d), p, p, p, 1.0, p, p, p, p, p, 16, p, 16, 1.0,
                    nul, nul, p, nul, p, 8, nul)
    assert st == 3 and "workspace" in msg
    kp = dsa.Dims(**{**d.as_dict(), "kpool": 4})
    st, msg = _call(lib.dsa_layer_forward, ctypes.byref(kp), p, p, p, 1.0, p, p, p, p, p, 16, p, 16, 1.0,
                    nul, nul, p, nul, p, 1 << 20, nul)
    assert st == 1 and "kpool" in msg
    # kpool entry points
    st, msg = _call(lib.dsa_pool_states, ctypes.byref(kp), p, p, nul, nul, 0.0, p, p, p, p, nul)
    assert st == 1 and "ln_eps" in msg
    narrow = dsa.Dims(**{**kp.as_dict(), "out_width": 4 * 4 + 2})
    st, msg = _call(lib.dsa_expand_selection, ctypes.byref(narrow), p, p, p, p, p, p, nul)
    assert st == 1 and "out_width" in msg
    f32 = dsa.Dims(**{**d.as_dict(), "dtype": dsa.F32})
    st, msg = _call(lib.dsa_absorb_q, ctypes.byref(f32), p, 16, p, 32, p, nul)
    assert st == 2 and "bf16" in msg
    st, msg = _call(lib.dsa_selftest_wait_timeout, 5, nul)
    assert st == 1
    # the key-ordered top-k validates like dsa_topk
    st, msg = _call(lib.dsa_topk_set, ctypes.byref(d), p, p, p, p, 0, p, nul, nul)
    assert st == 1 and "k must be" in msg
    st, msg = _call(lib.dsa_topk_set, ctypes.byref(d), p, nul, p, p, 4, p, nul, nul)
    assert st == 1 and "q_pos" in msg
    st, msg = _call(lib.dsa_absorb_out, ctypes.byref(f32), p, 32, p, 16, p, nul)
    assert st == 2 and "bf16" in msg
    # the allocation-free layer: dims checked, and a layer needing more than the fixed 16 MiB refused,
    # before any device call
    args = (p, p, p, 1.0, p, p, p, p, p, 16, p, 16, 1.0, nul, nul, p, nul, nul)
    st, msg = _call(lib.dsa_layer_forward_static, None, *args)
    assert st == 1 and "dims" in msg
    st, msg = _call(lib.dsa_layer_forward_static, ctypes.byref(dsa.Dims(batch=0, n_q=1, n_kv=1, top_k=1)), *args)
    assert st == 1
    big = dsa.Dims(**{**d.as_dict(), "n_q": 4096, "n_kv": 4096, "top_k": 2048})
    st, msg = _call(lib.dsa_layer_forward_static, ctypes.byref(big), *args)
    assert st == 3 and "16 MiB" in msg


def test_index_rotate_host_validation(lib):
    nul = None
    a = ctypes.c_void_p(256)  # 16-byte aligned, never dereferenced: validation fails first
    BF, F = dsa.BF16, dsa.F32

    def rot(n_rows=4, heads=2, dim=128, n_rope=64, theta=10000.0, ln=0, eps=0.0, pos=a, in_dt=BF, x=a,
            in_stride=256, out_dt=BF, out=a, out_stride=256, rows=nul, cap=4):
        return _call(lib.dsa_index_rotate, n_rows, heads, dim, n_rope, theta, ln, nul, nul, eps, 1, pos, in_dt, x,
                     in_stride, out_dt, out, out_stride, rows, cap, nul)

    assert rot(dim=96)[0] == 1 and "dim" in rot(dim=96)[1]
    assert rot(n_rope=62)[0] == 1                      # (n_rope/2) % (dim/32) != 0
    assert rot(n_rope=130)[0] == 1
    assert rot(n_rope=63, dim=32)[0] == 1              # odd
    assert rot(theta=0.0)[0] == 1 and "rope_theta" in rot(theta=0.0)[1]
    assert rot(ln=1, eps=0.0)[0] == 1 and "ln_eps" in rot(ln=1, eps=0.0)[1]
    assert rot(in_stride=200)[0] == 1 and "stride" in rot(in_stride=200)[1]
    assert rot(out_stride=258)[0] == 1                 # not a multiple of dim/32
    assert rot(x=ctypes.c_void_p(258))[0] == 1 and "aligned" in rot(x=ctypes.c_void_p(258))[1]
    assert rot(pos=nul)[0] == 1 and "pos" in rot(pos=nul)[1]
    assert rot(cap=3)[0] == 1 and "out_capacity" in rot(cap=3)[1]
    assert rot(heads=0)[0] == 1
    assert rot(in_dt=7)[0] == 1
    assert rot(n_rows=-1)[0] == 1
    assert rot(n_rows=0, x=nul, out=nul)[0] == 0       # nothing to do: no launch, no pointer read


def test_binding_raises_typed_errors(lib):
    with pytest.raises(dsa.DsaError) as ei:
        dsa._check(1, "dsa_topk")
    assert ei.value.name == "DSA_ERR_INVALID_ARGUMENT"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(dsa, "_lib", None)
    monkeypatch.setattr(dsa, "lib_path", lambda: str(tmp_path / "libdsa.so"))
    with pytest.raises(dsa.DsaLibraryError):
        dsa.lib()


def test_plain_c_program_links_and_calls_the_library(lib, tmp_path):
    """include/dsa.h is plain C99 and libdsa.so links into a C program (host-only calls, no GPU)."""
    src = tmp_path / "use_dsa.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "dsa.h"
int main(void) {
  dsa_dims d;
  memset(&d, 0, sizeof d);
  d.batch = 2; d.n_q = 3; d.n_kv = 100; d.top_k = 8;
  printf("%s|%s|%zu|", dsa_version(), dsa_status_string(DSA_ERR_TIMEOUT),
         dsa_workspace_size(&d, DSA_OP_LAYER_FORWARD));
  /* host validation: a NULL dims pointer is rejected before any launch */
  dsa_status s = dsa_index_scores(NULL, NULL, NULL, NULL, 1.0f, NULL, NULL, NULL, NULL, NULL);
  printf("%d|%s\n", (int)s, dsa_last_error());
  return s == DSA_ERR_INVALID_ARGUMENT ? 0 : 1;
}
''')
    exe = tmp_path / "use_dsa"
    pkg = os.path.dirname(dsa.lib_path())
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                         str(src), "-o", str(exe), "-L", pkg, "-ldsa", f"-Wl,-rpath,{pkg}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    version, status, ws, code, msg = run.stdout.strip().split("|")
    assert "sm_100a" in version and status == "DSA_ERR_TIMEOUT"
    assert int(ws) == dsa.workspace_size(dsa.Dims(batch=2, n_q=3, n_kv=100, top_k=8), dsa.OP_LAYER_FORWARD)
    assert int(code) == 1 and "dims" in msg


def test_kernel_policy_switch_returns_the_previous_setting(lib):
    prev = dsa.set_kernel_policy(1)
    try:
        assert dsa.set_kernel_policy(0) == 1
        assert dsa.set_kernel_policy(7) == 0      # anything but 1 selects the tensor-core family
        assert dsa.set_kernel_policy(1) == 0
        assert dsa.set_kernel_policy(1) == 1
    finally:
        dsa.set_kernel_policy(prev)


def test_binding_rejects_non_contiguous_dense_arguments():
    import torch
    with pytest.raises(ValueError, match="contiguous"):
        dsa._ptr(torch.zeros(4, 6).t())                 # transposed view for a dense argument
    with pytest.raises(ValueError, match="innermost"):
        dsa._ptr(torch.zeros(4, 6)[:, ::2], dense=False)  # strided rows still need unit inner stride
    with pytest.raises(ValueError, match="CUDA"):
        dsa._ptr(torch.zeros(4, 6)[:, :3], dense=False)   # a row-strided view passes the layout check
    assert dsa._ptr(None) is None
