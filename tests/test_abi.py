"""The C-ABI library loads, exports every entry point include/nosa.h declares,
and rejects bad host-visible arguments before touching the GPU (CPU only)."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nosa.h")


@pytest.fixture(scope="module")
def nosa():
    from long_context_decode_nosa_b200 import build
    build.build()
    from long_context_decode_nosa_b200 import nosa as m
    m.lib()
    return m


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"NOSA_API\s+[\w\s\*]*?\b(nosa_\w+)\s*\(", txt)))


def test_header_declares_the_path():
    names = _declared()
    for need in ("nosa_pool_append", "nosa_block_select", "nosa_sparse_decode",
                 "nosa_workspace_size", "nosa_read_device_status", "nosa_status_string"):
        assert need in names


def test_library_exports_every_declared_symbol(nosa):
    lib_path = nosa.LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (nosa_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        getattr(nosa.lib(), n)  # resolvable through ctypes too


def test_status_strings(nosa):
    for code in range(7):
        assert nosa.lib().nosa_status_string(code).decode()
    assert nosa.lib().nosa_status_string(99).decode() == "unknown status"


def test_workspace_size_host_only(nosa):
    p = nosa.params(16, 2, topk=64)
    n8 = nosa.workspace_size(p, 8, 16384)
    n16 = nosa.workspace_size(p, 16, 16384)
    assert n8 > 0 and n16 > n8 and n8 % 256 == 0
    bad = nosa.params(16, 3)
    assert nosa.lib().nosa_workspace_size(ctypes.byref(bad), 8, 16384) == 0


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, 2), ("pool_kernel", 16, 2), ("block_size", 128, 2), ("topk", 0, 2),
    ("local_blocks", 257, 2),
    ("num_kv_heads", 3, 1), ("local_blocks", -1, 1), ("softmax_scale", -1.0, 1),
])
def test_bad_params_rejected_before_any_launch(nosa, field, value, code):
    p = nosa.params(16, 2)
    setattr(p, field, value)
    rc = nosa.lib().nosa_sparse_decode(ctypes.byref(p), None, None, None, 0, None, None, 1, 16, None,
                                       None, None, None, None, 0, None)
    assert rc == code
    assert nosa.lib().nosa_last_error().decode()


def test_null_and_workspace_checks(nosa):
    p = nosa.params(16, 2)
    L = nosa.lib()
    # workspace missing
    rc = L.nosa_block_select(ctypes.byref(p), None, None, 1, None, 4, 1024, None, 0, None, None, 0,
                             None, None, None, 0, None)
    assert rc == nosa.NOSA_ERR_WORKSPACE
    # workspace too small (a host buffer stands in: the check fails before any use)
    buf = ctypes.create_string_buffer(1024 + 256)
    addr = (ctypes.addressof(buf) + 255) // 256 * 256
    rc = L.nosa_sparse_decode(ctypes.byref(p), None, None, None, 0, None, None, 4, 1024, None, None,
                              None, None, ctypes.c_void_p(addr), 1024, None)
    assert rc == nosa.NOSA_ERR_WORKSPACE
    # batch 0 is a no-op
    assert L.nosa_pool_append(ctypes.byref(p), None, None, 0, None, None, None, 0, None, 1, 1, None,
                              None, None, 0, None) == 0
    # k_new without v_new
    rc = L.nosa_pool_append(ctypes.byref(p), ctypes.c_void_p(256), None, 100, ctypes.c_void_p(256), None,
                            ctypes.c_void_p(256), 1, ctypes.c_void_p(256), 1, 1,
                            ctypes.c_void_p(256), None, None, 0, None)
    assert rc == nosa.NOSA_ERR_INVALID_ARG


# (entry point, index of batch (or total_q), index of max_seq_len or None, fixed args)
_DUMMY = ctypes.c_void_p(256)  # a page table that an empty batch never reads
_EMPTY_CALLS = [
    ("nosa_block_select", 5, 6, {}),
    ("nosa_sparse_decode", 7, 8, {}),
    ("nosa_sparse_decode_paged", 8, 9, {4: 1, 5: _DUMMY}),
    ("nosa_decode_step_device", 9, 10, {}),
    ("nosa_decode_step_device_paged", 10, 11, {6: 1, 7: _DUMMY}),
    ("nosa_decode_step", 10, 11, {}),
    ("nosa_decode_step_packed", 8, 9, {}),
    ("nosa_decode_step_device_noalloc", 9, 10, {}),
    ("nosa_pool_append_paged", 8, None, {3: 1, 4: _DUMMY, 10: 1, 11: 1}),
    ("nosa_sparse_prefill", 9, 10, {8: 1}),          # batch 1, total_q 0
    ("nosa_sparse_prefill_paged", 10, 11, {4: 1, 5: _DUMMY, 9: 1}),
]


@pytest.mark.parametrize("name,i_batch,i_len,extra", _EMPTY_CALLS, ids=[c[0] for c in _EMPTY_CALLS])
def test_empty_batch_is_a_no_op(nosa, name, i_batch, i_len, extra):
    """An empty batch (or no prefill rows) returns NOSA_OK before any check
    of the other buffers and before any CUDA call (none could run on this
    host); the paged calls still check the page pool's geometry (a page
    table pointer and at least one page)."""
    p = nosa.params(16, 2)
    fn = getattr(nosa.lib(), name)
    args = [ctypes.byref(p)] + [None if t is nosa._P else 0 for t in fn.argtypes[1:]]
    args[i_batch] = 0
    if i_len is not None:
        args[i_len] = 1024
    for k, v in extra.items():
        args[k] = v
    assert fn(*args) == nosa.NOSA_OK, nosa.lib().nosa_last_error().decode()


def test_noalloc_host_checks_come_first(nosa):
    """The scratch-free step runs the workspace entry point's host checks,
    and its own size check, before any CUDA call (none could run on this
    host): a NULL buffer and a batch beyond the built-in 8 MiB both return
    their codes with nothing enqueued."""
    p = nosa.params(16, 2, topk=64)
    fn = nosa.lib().nosa_decode_step_device_noalloc
    d = ctypes.c_void_p(256)
    rc = fn(ctypes.byref(p), None, None, None, d, d, 100, d, d, 4, 1024, d, 1, d, d, d, None, None)
    assert rc == nosa.NOSA_ERR_INVALID_ARG
    assert nosa.workspace_size(p, 64, 1 << 20) > 8 << 20
    rc = fn(ctypes.byref(p), d, None, None, d, d, 1 << 30, d, d, 64, 1 << 20, d, 1, d, d, d, None, None)
    assert rc == nosa.NOSA_ERR_WORKSPACE
    assert "8388608" in nosa.lib().nosa_last_error().decode()


_C_CLIENT = r"""
#include <stdio.h>
#include "nosa.h"
int main(void) {
  nosa_params p;
  nosa_default_params(&p);
  p.num_q_heads = 16;
  p.num_kv_heads = 2;
  size_t ws = nosa_workspace_size(&p, 8, 16384);
  printf("%zu|%s|%d\n", ws, nosa_status_string(NOSA_ERR_INVALID_ARG),
         nosa_block_select(&p, NULL, NULL, 0, NULL, 0, 1024, NULL, 0, NULL, NULL, 0, NULL, NULL, NULL, 0, NULL));
  return ws == 0;
}
"""


def test_plain_c_client(nosa, tmp_path):
    """The header compiles as strict C99 and a plain C program links against
    the library and calls it (host-only calls: no GPU here), with no Python
    or PyTorch involved."""
    import shutil
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(_C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(nosa.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.dirname(HEADER), str(src),
                    "-L", libdir, "-lnosa_b200", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.strip().split("|")
    p = nosa.params(16, 2)
    assert int(out[0]) == nosa.lib().nosa_workspace_size(ctypes.byref(p), 8, 16384) > 0
    assert out[1] == nosa.lib().nosa_status_string(nosa.NOSA_ERR_INVALID_ARG).decode()
    assert int(out[2]) == nosa.NOSA_OK  # batch 0
