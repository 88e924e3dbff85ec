"""The C-ABI library loads and exports every symbol include/kvc.h declares, and the
Python structs match the C layout (checked by compiling the header with gcc). No GPU
compute is called here."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^KVC_API\s+[\w\s\*]+?\b(kvc_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    import transformer_kv_cache_b200 as kvc
    names = _declared()
    assert len(names) >= 18
    lib = ctypes.CDLL(kvc.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(kvc.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", kvc.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted(set(re.findall(r" T (kvc_\w+)", out)))
    assert exported == names, "the library exports exactly the declared entry points"


def test_struct_layout_matches_header():
    import transformer_kv_cache_b200 as kvc
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "kvc.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(kvc_config), sizeof(kvc_info), offsetof(kvc_config, softmax_scale),
         offsetof(kvc_config, kv_splits), offsetof(kvc_config, reserved), offsetof(kvc_info, device_error));
  return 0;
}'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "t")
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True).stdout.split()]
    C, I = kvc.kvc_config, kvc.kvc_info
    assert vals == [ctypes.sizeof(C), ctypes.sizeof(I), C.softmax_scale.offset, C.kv_splits.offset,
                    C.reserved.offset, I.device_error.offset]


def test_host_only_calls_and_config_validation():
    import transformer_kv_cache_b200 as kvc
    assert kvc.kvc_version() == 1
    assert kvc.kvc_status_string(5) == "KVC_ERR_BUDGET"
    bad = kvc.make_config(1, 2, 48, 10, 1, 8, 2, 0)       # head_dim 48 is rejected before any CUDA call
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_create(bad, stream=0)
    assert e.value.status_name == "KVC_ERR_ARG"
    bad = kvc.make_config(1, 2, 64, 10, 1, 8, 2, 0, budget_tokens=100)   # window and budget together
    with pytest.raises(kvc.KVCError):
        kvc.kvc_create(bad, stream=0)
