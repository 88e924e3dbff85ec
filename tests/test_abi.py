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
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(kvc_config), sizeof(kvc_info), offsetof(kvc_config, softmax_scale),
         offsetof(kvc_config, kv_splits), offsetof(kvc_config, model_heads), offsetof(kvc_config, head_begin),
         offsetof(kvc_config, reserved), offsetof(kvc_info, device_error));
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
                    C.model_heads.offset, C.head_begin.offset, C.reserved.offset, I.device_error.offset]


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


# Each rule of kvc_create's argument check, one at a time: the unmodified workload config
# passes the check (without a GPU it then fails at its first device allocation, never with
# KVC_ERR_ARG; with one it is created and destroyed), and the one change makes it
# KVC_ERR_ARG before any CUDA call.
CONFIG_RULES = [
    ("vggt_518x378", dict(head_dim=48), "head dim outside 16/32/64/128"),
    ("vggt_518x378", dict(num_special_tokens=1005), "more special tokens than a frame holds"),
    ("vggt_518x378", dict(io_dtype="f32"), "bf16 storage under fp32 inputs"),
    ("vggt_518x378", dict(softmax_scale=float("nan")), "softmax scale not finite"),
    ("vggt_518x378", dict(softmax_scale=0.0), "softmax scale not positive"),
    ("vggt_518x378", dict(kv_splits=-1), "negative KV split count"),
    ("vggt_518x378", dict(budget_tokens=16384), "window and token budget together"),
    ("vggt_518x378", dict(window_frames=0, max_frames=0), "no window, budget or frame cap"),
    ("vggt_518x378", dict(fp8_dim_adaptive=1), "dimension-adaptive scales on bf16 storage"),
    ("vggt_518x378_special", dict(special_frames=-1), "negative special-frame cap"),
    ("vggt_518x378_special", dict(window_frames=0, max_frames=100), "special tokens without a window"),
    ("vggt_518x518_fp8", dict(io_dtype="f32"), "FP8 storage under fp32 inputs"),
    ("vggt_518x518_fp8", dict(page_size=64), "FP8 page-head block over 2 KB"),
    ("vggt_518x518_fp8da", dict(fp8_dim_adaptive=2), "unknown quantisation mode"),
    ("vggt_518x518_fp8da", dict(page_size=8), "dimension-adaptive FP8 off the 16 x 64 block"),
    ("vggt_budget_16k", dict(kv_dtype="fp8_e4m3"), "token budget on FP8 storage"),
    ("vggt_budget_16k", dict(keep_frac=0.0), "empty keep tier"),
    ("vggt_budget_16k", dict(rank_window=0), "empty rank window"),
    ("vggt_budget_16k", dict(lam=-0.5), "negative consistency weight"),
    ("vggt_infinite_12l", dict(page_size=8), "rolling memory off the 16-slot page"),
    ("vggt_infinite_12l", dict(diversity_budget=1100), "more candidates than the pruning cluster holds"),
    ("vggt_infinite_12l", dict(diversity_budget=-1), "negative diversity budget"),
    ("vggt_infinite_12l", dict(window_frames=64), "rolling memory with a window"),
    ("vggt_518x378", dict(window_frames=(1 << 24) + 1), "window past its cap"),
    ("vggt_518x378", dict(window_frames=0, max_frames=(1 << 24) + 1), "frame cap past its cap"),
    ("vggt_518x378", dict(window_frames=0, max_frames=200_000), "pool rows past the int row index"),
    ("vggt_518x378", dict(tokens_per_frame=(1 << 24) + 1), "frame past the token cap"),
    ("vggt_518x378", dict(head_begin=2**31 - 2), "head range overflowing int"),
    ("vggt_518x378", dict(io_dtype="f32", kv_dtype="f32", tokens_per_frame=1 << 22),
     "frame past the int element index"),
    ("vggt_518x378", dict(io_dtype="f32", kv_dtype="f32", page_size=1 << 16, num_heads=1 << 10),
     "page past the int element index"),
    ("vggt_infinite_12l", dict(diversity_budget=2**31 - 1), "diversity budget overflowing int"),
]


@pytest.mark.parametrize("workload,change,why", CONFIG_RULES, ids=[r[2] for r in CONFIG_RULES])
def test_config_rule_rejected_before_any_cuda_call(workload, change, why):
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS
    wl = WORKLOADS[workload]
    try:
        h = kvc.kvc_create(kvc.config_from_workload(wl), stream=0)
    except kvc.KVCError as e:
        assert e.status_name != "KVC_ERR_ARG", f"base config of {workload} fails the argument check"
    else:
        kvc.kvc_destroy(h)                      # a device is present and the base was created
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_create(kvc.config_from_workload(wl, **change), stream=0)
    assert e.value.status_name == "KVC_ERR_ARG", why


def test_reserved_config_words_must_be_zero():
    import transformer_kv_cache_b200 as kvc
    from kvc_streams import WORKLOADS
    cfg = kvc.config_from_workload(WORKLOADS["vggt_518x378"])
    cfg.reserved[1] = 7
    with pytest.raises(kvc.KVCError) as e:
        kvc.kvc_create(cfg, stream=0)
    assert e.value.status_name == "KVC_ERR_ARG"


def test_null_handle_is_rejected_by_every_entry_point():
    """Host-only: every call that takes a cache handle returns KVC_ERR_ARG for NULL (no
    dereference, no CUDA call); kvc_destroy(NULL) is a no-op; the allocation-free entry
    point rejects NULL device pointers."""
    import transformer_kv_cache_b200 as kvc
    lib = kvc._lib
    no_handle = {"kvc_create", "kvc_status_string", "kvc_version", "kvc_debug_fail_allocs",
                 "kvc_attend_paged_noalloc", "kvc_destroy", "kvc_last_error"}

    def zero_args(fn):
        out = []
        for t in fn.argtypes:
            if t in (ctypes.c_float, ctypes.c_double):
                out.append(0.0)
            elif t in (ctypes.c_int32, ctypes.c_int64, ctypes.c_int):
                out.append(0)
            else:
                out.append(None)                    # handle and every pointer
        return out

    checked = 0
    for name in kvc.EXPORTS:
        if name in no_handle:
            continue
        fn = getattr(lib, name)
        assert fn.argtypes, f"{name} has no declared signature in the binding"
        assert fn(*zero_args(fn)) == 1, name       # KVC_ERR_ARG
        checked += 1
    assert checked >= 20
    assert lib.kvc_destroy(None) == 0
    assert ctypes.string_at(lib.kvc_last_error(None)) == b"null cache"
    fn = lib.kvc_attend_paged_noalloc
    assert fn(*zero_args(fn)) == 1


# The allocation-free entry point's host checks, one rule at a time, with fake 16-byte
# aligned device addresses. Run only where no GPU is present: a rule that stopped
# rejecting then ends at the first CUDA call (KVC_ERR_CUDA) instead of launching over
# addresses that do not exist.
NOALLOC_BASE = dict(q=0x10000, o=0x20000, k_pool=0x30000, v_pool=0x40000, pool_pages=64, page_table=0x50000,
                    n_pages=8, tokens=300, num_heads=4, head_dim=64, page_size=16, softmax_scale=0.125,
                    kv_splits=1)
NOALLOC_RULES = [
    (dict(head_dim=32), "head dim other than 64"),
    (dict(page_size=8), "page size other than 16"),
    (dict(tokens=0), "no query rows"),
    (dict(num_heads=0), "no heads"),
    (dict(n_pages=0), "no pages"),
    (dict(pool_pages=0), "empty pool"),
    (dict(softmax_scale=0.0), "scale not positive"),
    (dict(softmax_scale=float("nan")), "scale NaN"),
    (dict(softmax_scale=float("inf")), "scale infinite"),
    (dict(kv_splits=0), "no KV split"),
    (dict(q=0x10008), "Q not 16-byte aligned"),
    (dict(page_table=0x50004), "page table not 16-byte aligned"),
    (dict(pool_pages=2**31 // (4 * 16) + 1), "pool rows past the int row index"),
    (dict(tokens=1025 * 128), "more piece counters than the array holds"),
]


@pytest.mark.parametrize("change,why", NOALLOC_RULES, ids=[r[1] for r in NOALLOC_RULES])
def test_noalloc_rule_rejected_before_any_cuda_call(change, why):
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device addresses: host checks only, on a host without a GPU")
    import transformer_kv_cache_b200 as kvc
    fn = kvc._lib.kvc_attend_paged_noalloc

    def call(**over):
        a = dict(NOALLOC_BASE, **over)
        return fn(a["q"], a["o"], a["k_pool"], a["v_pool"], a["pool_pages"], a["page_table"], a["n_pages"],
                  a["tokens"], a["num_heads"], a["head_dim"], a["page_size"], a["softmax_scale"],
                  a["kv_splits"], None)

    assert call() == 3, "the base call passes the host checks and stops at the first CUDA call"
    assert call(**change) == 1, why             # KVC_ERR_ARG


def test_plain_c_program_links_and_calls_the_library():
    """A C99 program compiled against include/kvc.h and linked with libkvc.so: the host-only
    calls work without Python (version, status strings, argument rejection, NULL handles)."""
    import transformer_kv_cache_b200 as kvc
    prog = r'''
#include <stdio.h>
#include <string.h>
#include "kvc.h"
int main(void) {
  kvc_config cfg;
  kvc_cache* c = (kvc_cache*)1;
  memset(&cfg, 0, sizeof(cfg));
  cfg.num_layers = 1; cfg.num_heads = 16; cfg.head_dim = 48;   /* head dim 48 is rejected */
  cfg.tokens_per_frame = 1004; cfg.page_size = 16; cfg.window_frames = 64;
  cfg.io_dtype = KVC_BF16; cfg.kv_dtype = KVC_BF16; cfg.softmax_scale = 0.125f;
  kvc_status st = kvc_create(&cfg, NULL, &c);
  printf("%d %d %s %d %d %s\n", (int)kvc_version(), (int)st, kvc_status_string(st), c == NULL,
         (int)kvc_attend(NULL, 0, NULL, NULL), kvc_last_error(NULL));
  return 0;
}'''
    lib_dir = os.path.dirname(kvc.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "use_kvc.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "use_kvc")
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe,
                        "-L", lib_dir, "-lkvc", "-Wl,-rpath," + lib_dir], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    assert out == ["1", "1", "KVC_ERR_ARG", "1", "1", "null", "cache"]


def test_binding_refuses_host_buffers_for_device_arguments():
    """The binding hands the library only CUDA tensors (or explicit addresses) where a
    kernel reads or writes: a CPU tensor or numpy array raises before any C call."""
    import numpy as np
    import torch
    import transformer_kv_cache_b200 as kvc
    host_t, host_np = torch.zeros(16), np.zeros(16, np.float32)
    for bad in (host_t, host_np):
        with pytest.raises(TypeError):
            kvc.kvc_attend(0, 0, bad, bad)
        with pytest.raises(TypeError):
            kvc.kvc_append_frame(0, 0, 0, bad, bad)
        with pytest.raises(TypeError):
            kvc.kvc_attend_all(0, [bad], [bad])
        with pytest.raises(TypeError):
            kvc.kvc_compress(0, 0, bad)
        with pytest.raises(TypeError):
            kvc.kvc_attend_paged_noalloc(bad, bad, bad, bad, 1, bad, 1, 1, 1, 64, 16, 0.125)


@pytest.mark.parametrize("compiler,std,ext", [("gcc", "c99", "c"), ("g++", "c++17", "cpp")])
def test_header_compiles_without_warnings(compiler, std, ext):
    """include/kvc.h is plain C: it compiles warning-free under strict C99 and C++17."""
    src = '#include "kvc.h"\nint main(void) { kvc_config c; (void)c; return (int)kvc_version(); }\n'
    with tempfile.TemporaryDirectory() as d:
        f = os.path.join(d, "hdr." + ext)
        open(f, "w").write(src)
        subprocess.run([compiler, "-std=" + std, "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), "-c", f, "-o", os.path.join(d, "hdr.o")], check=True)
