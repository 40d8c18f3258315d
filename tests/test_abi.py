"""The C ABI library builds, loads without a GPU, and exports every declared symbol."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kv_\w+|paged_attention_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kv_cache_append", "paged_attention_decode", "paged_attention_workspace_size",
                     "kv_pool_create", "kv_pool_alloc", "kv_pool_free", "kv_pool_incref"):
        assert required in names


def test_library_exports_every_declared_symbol(pkv):
    lib = ctypes.CDLL(pkv.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in pagedkv.h but not exported"


def test_binding_covers_every_declared_symbol(pkv):
    assert set(declared_functions()) == set(pkv.EXPORTED)


def test_only_abi_symbols_are_exported(pkv):
    out = subprocess.run(["nm", "-D", "--defined-only", pkv.LIB_PATH], capture_output=True, text=True).stdout
    ours = {l.split()[-1] for l in out.splitlines() if re.search(r"\b(kv_|paged_attention_)", l)}
    assert ours == set(declared_functions())


def test_library_is_built_for_sm100a(pkv):
    # the build flags are the contract; check them without reading the binary
    import runpy
    flags = runpy.run_path(os.path.join(ROOT, "paged_kv_cache_470_b200", "build.py"))["NVCC_FLAGS"]
    assert "arch=compute_100a,code=sm_100a" in " ".join(flags)


def test_host_argument_checks_need_no_gpu(pkv):
    lib = ctypes.CDLL(pkv.LIB_PATH)
    lib.kv_cache_append.restype = ctypes.c_int
    # D = 96 is not supported: rejected on the host before any CUDA call
    rc = lib.kv_cache_append(None, None, None, None, None, 1, 1, 1, 96, 0, None, None)
    assert rc == pkv.KV_ERR_ARG
    assert pkv.set_option(pkv.KV_OPT_COMPUTE, 0) is None
    assert lib.kv_decode_set_option(99, 0) == pkv.KV_ERR_ARG


def test_option_ranges_need_no_gpu(pkv):
    """Every switch takes its documented values, keeps them, and refuses the rest."""
    lib = ctypes.CDLL(pkv.LIB_PATH)
    lib.kv_decode_set_option.restype = ctypes.c_int
    lib.kv_decode_get_option.restype = ctypes.c_int
    cases = {pkv.KV_OPT_PREFILL_PATH: ([0, 1, 2, 3], [-1, 4]),
             pkv.KV_OPT_TEST_SLOW_SOFTMAX: ([0, 1], [-1, 2]),
             pkv.KV_OPT_TEST_DROP_LOAD: ([0, 5], [-1]),
             pkv.KV_OPT_ITEM_COST: ([-1, 0, 64], [-2, 65]),
             pkv.KV_OPT_OUT_F32: ([0, 1], [-1, 2]),
             pkv.KV_OPT_L2_POLICY: ([0, 1, 2, 3], [-1, 4]),
             pkv.KV_OPT_EARLY_LOADS: ([0, 1], [-1, 2])}
    for key, (good, bad) in cases.items():
        before = lib.kv_decode_get_option(key)
        for v in good:
            assert lib.kv_decode_set_option(key, v) == pkv.KV_OK
            assert lib.kv_decode_get_option(key) == v
        for v in bad:
            assert lib.kv_decode_set_option(key, v) == pkv.KV_ERR_ARG
            assert lib.kv_decode_get_option(key) == good[-1]
        assert lib.kv_decode_set_option(key, before) == pkv.KV_OK


def test_binding_has_every_call_under_its_own_name(pkv):
    """Every call the header declares is a Python function of the same name."""
    for name in declared_functions():
        assert callable(getattr(pkv, name, None)), f"{name} has no same-named binding"


def test_pool_calls_by_their_abi_names_need_no_gpu(pkv):
    import torch
    pool = pkv.kv_pool_create(8)
    ids = pkv.kv_pool_alloc(pool, 3)
    assert pkv.kv_pool_num_free(pool) == 5 and pkv.kv_pool_num_blocks(pool) == 8
    child = pkv.kv_pool_fork(pool, ids[:2])
    assert child == ids[:2] and pkv.kv_pool_refcount(pool, ids[0]) == 2
    pkv.kv_pool_incref(pool, [ids[2]])
    pkv.kv_pool_free(pool, [ids[2], ids[2]])
    assert pkv.kv_pool_refcount(pool, ids[2]) == 0 and pkv.kv_pool_num_free(pool) == 6
    # one step of bookkeeping for a sequence with 16 tokens: it needs a second block
    tables = torch.full((1, 4), -1, dtype=torch.int32)
    tables[0, 0] = ids[1]
    lens = torch.tensor([16], dtype=torch.int32)
    slots = torch.zeros(1, dtype=torch.int64)
    pkv.kv_pool_append_slots(pool, tables, lens, slots)
    assert int(lens[0]) == 17 and int(tables[0, 1]) >= 0 and int(slots[0]) == int(tables[0, 1]) * 16
    src, dst = pkv.kv_pool_append_slots_cow(pool, tables, lens, slots)
    assert (src, dst) == ([], []) and int(lens[0]) == 18
    assert pkv.kv_decode_get_option(pkv.KV_OPT_PREFILL_PATH) == pkv.get_option(pkv.KV_OPT_PREFILL_PATH)
    pkv.kv_pool_destroy(pool)


C_CLIENT = r"""
#include "pagedkv.h"
#include <stdio.h>
int main(void) {
    void *pool = 0;
    int32_t ids[3], child[2];
    if (kv_pool_create(8, &pool) != KV_OK) return 1;
    if (kv_pool_alloc(pool, 3, ids) != KV_OK || kv_pool_num_free(pool) != 5) return 2;
    if (kv_pool_fork(pool, ids, 2, child) != KV_OK || kv_pool_refcount(pool, ids[0]) != 2) return 3;
    if (kv_pool_free(pool, child, 2) != KV_OK || kv_pool_free(pool, ids, 3) != KV_OK) return 4;
    if (kv_pool_num_free(pool) != 8 || kv_pool_alloc(pool, 9, ids) != KV_ERR_OOM) return 5;
    kv_pool_destroy(pool);
    if (kv_decode_set_option(99, 0) != KV_ERR_ARG) return 6;
    printf("c client ok\n");
    return 0;
}
"""


def test_a_plain_c_program_uses_the_library(pkv, tmp_path):
    """The boundary is a C ABI: a C99 program includes the header, links the library and calls it."""
    import shutil
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(pkv.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-lpagedkv", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "c client ok", (out.returncode, out.stdout, out.stderr)


def test_importing_the_package_maps_no_library():
    """The package's input generator can be imported by code that must not load the CUDA library (the oracle's
    timed arm): the library is mapped by the first call that needs it."""
    code = ("import sys; sys.path.insert(0, %r); import paged_kv_cache_470_b200 as p; "
            "from paged_kv_cache_470_b200 import workloads; "
            "maps = open('/proc/self/maps').read(); assert 'libpagedkv' not in maps, 'mapped at import'; "
            "p.load(); assert 'libpagedkv' in open('/proc/self/maps').read(); print('ok')") % ROOT
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stderr


def test_multi_layer_checks_need_no_gpu(pkv):
    """paged_attention_decode_layers refuses bad layer arguments on the host, before any CUDA call."""
    lib = ctypes.CDLL(pkv.LIB_PATH)
    f = lib.paged_attention_decode_layers
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, ctypes.c_size_t, I, P, P, I, P, I, I, I, I, I, ctypes.c_float, I, P,
                  ctypes.c_size_t, P]
    f.restype = I
    fake = 1 << 20   # an aligned non-null address; nothing is dereferenced before the checks fail
    good = dict(out=fake, q=fake, kn=None, vn=None, kc=fake, vc=fake, stride=4 * 16 * 4 * 64, L=2, slots=None,
                tables=fake, W=4, lens=fake, B=3, nb=4, Hq=8, Hkv=4, D=64, scale=0.1, dtype=0, ws=fake,
                wsb=1 << 30)

    def call(**kw):
        a = dict(good, **kw)
        return f(a["out"], a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["stride"], a["L"], a["slots"],
                 a["tables"], a["W"], a["lens"], a["B"], a["nb"], a["Hq"], a["Hkv"], a["D"], a["scale"],
                 a["dtype"], a["ws"], a["wsb"], None)
    assert call(L=0) == pkv.KV_ERR_ARG                           # no layer
    assert call(stride=4 * 16 * 4 * 64 - 8) == pkv.KV_ERR_ARG    # layers would overlap
    assert call(stride=4 * 16 * 4 * 64 + 4) == pkv.KV_ERR_ARG    # not a multiple of 16 bytes
    assert call(kn=fake) == pkv.KV_ERR_ARG                       # new K rows without V rows and slots
    assert call(kn=fake, vn=fake, slots=fake + 4) == pkv.KV_ERR_ARG   # misaligned slots
    assert call(B=0) == pkv.KV_OK                                # nothing to do


def test_prefill_checks_need_no_gpu(pkv):
    """paged_attention_prefill refuses bad arguments on the host, before any CUDA call, including a batch whose
    rows would need more than 65,535 CTAs along the default kernel's second grid dimension (256 rows each)."""
    lib = ctypes.CDLL(pkv.LIB_PATH)
    f = lib.paged_attention_prefill
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, ctypes.c_float, I, P, P]
    f.restype = I
    fake = 1 << 20   # an aligned non-null address; nothing is dereferenced before the checks fail
    good = dict(out=fake, q=fake, kc=fake, vc=fake, tables=fake, W=4, lens=fake, qs=fake, B=3, maxq=32, nb=4,
                Hq=64, Hkv=8, D=128, scale=0.1, dtype=0)

    def call(**kw):
        a = dict(good, **kw)
        return f(a["out"], a["q"], a["kc"], a["vc"], a["tables"], a["W"], a["lens"], a["qs"], a["B"], a["maxq"],
                 a["nb"], a["Hq"], a["Hkv"], a["D"], a["scale"], a["dtype"], None, None)
    assert pkv.get_option(pkv.KV_OPT_PREFILL_PATH) == 0
    assert call(D=96) == pkv.KV_ERR_ARG                  # head dimension
    assert call(Hkv=6) == pkv.KV_ERR_ARG                 # Hq not a multiple of Hkv
    assert call(scale=0.0) == pkv.KV_ERR_ARG             # scale must be positive
    assert call(dtype=2) == pkv.KV_ERR_ARG               # element type
    assert call(q=fake + 8) == pkv.KV_ERR_ARG            # misaligned rows
    assert call(qs=None) == pkv.KV_ERR_ARG               # no query offsets
    # 8 query heads per kv head: ceil(maxq * 8 / 256) tile groups must stay <= 65535
    assert call(maxq=65535 * 32 + 1) == pkv.KV_ERR_ARG
    assert call(B=0) == pkv.KV_OK                        # nothing to do
    assert call(maxq=0) == pkv.KV_OK
