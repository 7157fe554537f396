"""The C-ABI library loads, exports every symbol the header declares, and
rejects invalid arguments on the host before any launch (no GPU needed)."""

from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "paged_kv_attention_35_b200", "libpagedattn.so")


@pytest.fixture(scope="module")
def ops():
    if not os.path.exists(LIB):
        from paged_kv_attention_35_b200.build import build
        build()
    from paged_kv_attention_35_b200 import ops as o
    return o


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M))
    return names


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ["pa_store_kvcache", "pa_decode", "pa_decode_workspace_size", "pa_prefill_varlen",
              "pa_status_string", "pa_last_error_message"]:
        assert n in names


def test_every_declared_symbol_is_exported(ops):
    lib = ctypes.CDLL(LIB)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert set(ops.SIGNATURES) >= declared_symbols()


def test_status_strings(ops):
    lib = ops.lib()
    for code, name in ops.STATUS.items():
        assert lib.pa_status_string(code).decode() == name
    assert lib.pa_status_string(99).decode() == "PA_ERR_UNKNOWN"
    assert "sm_100a" in ops.version()


def _store(ops, **kw):
    a = dict(key=16, value=16, ks=1024, vs=1024, kc=256, vc=256, slots=64, n=4, hkv=8, d=128,
             num_slots=4096, dtype=0, flag=None)
    a.update(kw)
    return ops.lib().pa_store_kvcache(a["key"], a["value"], a["ks"], a["vs"], a["kc"], a["vc"],
                                      a["slots"], a["n"], a["hkv"], a["d"], a["num_slots"], a["dtype"],
                                      a["flag"], None)


def test_store_validation(ops):
    assert _store(ops, dtype=1) == 2
    assert _store(ops, n=-1) == 1
    assert _store(ops, n=0, key=None) == 0                  # empty step: no-op, nothing touched
    assert _store(ops, key=None) == 1
    assert _store(ops, key=18) == 1                         # misaligned
    assert _store(ops, ks=100) == 1                         # stride < row
    assert _store(ops, ks=1028) == 1                        # stride not 16-byte multiple
    assert _store(ops, hkv=1, d=4) == 2                     # 8-byte rows
    assert _store(ops, num_slots=0) == 1
    assert b"num_slots" in ops.lib().pa_last_error_message()


def _decode(ops, **kw):
    a = dict(out=256, q=256, qs=2048, kc=256, vc=256, bt=64, mb=16, cl=64, B=4, maxc=4096, hq=16,
             hkv=8, d=128, bs=256, nb=64, scale=0.088, part=0, ws=None, wsb=0, dtype=0, flag=None)
    a.update(kw)
    return ops.lib().pa_decode(a["out"], a["q"], a["qs"], a["kc"], a["vc"], a["bt"], a["mb"], a["cl"],
                               a["B"], a["maxc"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"],
                               a["scale"], a["part"], a["ws"], a["wsb"], a["dtype"], a["flag"], None)


def test_decode_validation(ops):
    assert _decode(ops, hq=12, hkv=8) == 1                  # group not integral
    assert _decode(ops, d=96) == 2
    assert _decode(ops, bs=48) == 2
    assert _decode(ops, bs=8) == 2
    assert _decode(ops, kc=None) == 1
    assert _decode(ops, q=258) == 1
    assert _decode(ops, mb=4) == 1                          # 4*256 < max_context_len
    assert _decode(ops, scale=0.0) == 1
    assert _decode(ops, scale=float("nan")) == 1
    assert _decode(ops, part=100) == 1
    assert _decode(ops, B=0) == 0                           # nothing to do
    assert _decode(ops, dtype=3) == 2
    st = _decode(ops)                                       # needs a workspace
    assert st == 3
    msg = ops.lib().pa_last_error_message().decode()
    assert "workspace" in msg
    need = ops.decode_workspace_size(4, 16, 8, 128, 4096)
    assert need > 0
    assert _decode(ops, ws=257, wsb=need) == 3              # misaligned workspace


def test_workspace_size_rule(ops):
    # no split when the context fits one partition
    assert ops.decode_workspace_size(4, 16, 8, 128, 256, 256) == 0
    ws = ops.decode_workspace_size(4, 16, 8, 128, 1024, 256)
    rows = 4 * 16 * 4
    assert ws >= rows * 128 * 4 + rows * 2 * 4
    assert ops.decode_workspace_size(0, 16, 8, 128, 1024, 0) == 0


def _prefill(ops, **kw):
    a = dict(out=256, q=256, qs=3584, kc=256, vc=256, cq=64, ck=64, mq=128, mk=256, tq=128, bt=64,
             mb=4, B=2, hq=28, hkv=4, d=128, bs=256, nb=64, scale=0.088, dtype=0, flag=None)
    a.update(kw)
    return ops.lib().pa_prefill_varlen(a["out"], a["q"], a["qs"], a["kc"], a["vc"], a["cq"], a["ck"],
                                       a["mq"], a["mk"], a["tq"], a["bt"], a["mb"], a["B"], a["hq"],
                                       a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["dtype"],
                                       a["flag"], None)


def test_prefill_validation(ops):
    assert _prefill(ops, mq=300, mk=256) == 1               # max_seqlen_q > max_seqlen_k
    assert _prefill(ops, mb=0) == 1
    assert _prefill(ops, qs=100) == 1
    assert _prefill(ops, cq=None) == 1
    assert _prefill(ops, hq=6, hkv=4) == 1
    assert _prefill(ops, B=0) == 0
    assert _prefill(ops, tq=0) == 0


def _prefill_store(ops, **kw):
    a = dict(out=256, q=256, qs=3584, key=512, value=512, ks=512, vs=512, slots=64, kc=256, vc=256,
             cq=64, ck=64, mq=128, mk=256, tq=128, bt=64, mb=4, B=2, hq=28, hkv=4, d=128, bs=256,
             nb=64, scale=0.088, dtype=0, flag=None)
    a.update(kw)
    return ops.lib().pa_prefill_store(a["out"], a["q"], a["qs"], a["key"], a["value"], a["ks"],
                                      a["vs"], a["slots"], a["kc"], a["vc"], a["cq"], a["ck"], a["mq"],
                                      a["mk"], a["tq"], a["bt"], a["mb"], a["B"], a["hq"], a["hkv"],
                                      a["d"], a["bs"], a["nb"], a["scale"], a["dtype"], a["flag"], None)


def test_prefill_store_validation(ops):
    assert _prefill_store(ops, slots=None) == 1               # the store needs its slots
    assert _prefill_store(ops, key=None) == 1
    assert _prefill_store(ops, value=520) == 1                # misaligned new rows
    assert _prefill_store(ops, ks=256) == 1                   # stride < Hkv*D
    assert _prefill_store(ops, vs=516) == 1                   # stride not a multiple of 8
    # the prefill checks still apply
    assert _prefill_store(ops, mq=300, mk=256) == 1
    assert _prefill_store(ops, hq=6, hkv=4) == 1
    assert _prefill_store(ops, B=0) == 0                      # nothing to do
    assert "" == ops.lib().pa_last_error_message().decode()


def test_python_binding_refuses_cpu_tensors(ops):
    import torch
    x = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    pool = torch.zeros(4, 16, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        ops.store_kvcache(x, x, pool, pool, torch.zeros(2, dtype=torch.int32))


def _decode_store(ops, **kw):
    a = dict(out=256, q=256, qs=2048, key=512, value=512, ks=1024, vs=1024, slots=64, kc=256, vc=256,
             bt=64, mb=16, cl=64, B=4, maxc=4096, hq=16, hkv=8, d=128, bs=256, nb=64, scale=0.088,
             part=0, ws=None, wsb=0, dtype=0, flag=None)
    a.update(kw)
    return ops.lib().pa_decode_store(a["out"], a["q"], a["qs"], a["key"], a["value"], a["ks"], a["vs"],
                                     a["slots"], a["kc"], a["vc"], a["bt"], a["mb"], a["cl"], a["B"],
                                     a["maxc"], a["hq"], a["hkv"], a["d"], a["bs"], a["nb"], a["scale"],
                                     a["part"], a["ws"], a["wsb"], a["dtype"], a["flag"], None)


def test_decode_store_validation(ops):
    assert _decode_store(ops, key=None) == 1                 # new rows missing
    assert _decode_store(ops, slots=None) == 1
    assert _decode_store(ops, value=520) == 1                # misaligned
    assert _decode_store(ops, ks=100) == 1                   # stride < Hkv*D
    assert _decode_store(ops, vs=1028) == 1                  # stride not a multiple of 8
    assert _decode_store(ops, B=0, key=None, slots=None) == 0   # empty step: nothing to do
    # the decode checks still apply, and a missing workspace is reported as for pa_decode
    assert _decode_store(ops, hq=12, hkv=8) == 1
    assert _decode_store(ops) == 3
    assert "workspace" in ops.lib().pa_last_error_message().decode()


def test_selftest_validation(ops):
    assert ops.lib().pa_selftest_wait_timeout(None, 0, None, None) == 1
    assert ops.lib().pa_selftest_wait_timeout(None, 3_000_000, None, None) == 1


def test_header_is_plain_c_and_links(ops, tmp_path):
    """The boundary needs no Python or C++: a strict C99 program includes the header, links
    the library, and gets a workspace size and a host-side argument error back from it."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "consumer.c"
    src.write_text(r'''
#include "pagedattn.h"
#include <stdio.h>
int main(void) {
  size_t need = pa_decode_workspace_size(256, 28, 4, 128, 4096, 0);
  pa_status s = pa_store_kvcache(0, 0, 0, 0, 0, 0, 0, 1, 4, 128, 1024, PA_BF16, 0, 0);
  printf("%zu %d %s\n", need, (int)s, pa_status_string(s));
  return s == PA_OK;
}
''')
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(LIB)
    subprocess.run([cc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lpagedattn", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    need, code, name = out.stdout.split()
    assert int(need) > 0
    assert ops.STATUS[int(code)] == "PA_ERR_INVALID_ARG" == name
