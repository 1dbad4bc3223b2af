"""The C-ABI library loads and exports every function that include/ckv.h declares.

These tests run without a GPU. They make no compute call, only the host-side ones that
need no device (defaults, error strings, argument checks).
"""
import ctypes as C
import os
import re
import subprocess

import pytest

import recallable_kv_cache_cosine_b200 as ckv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ckv.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)
    return sorted({n for n in names if n not in ("if", "defined")})


@pytest.fixture(scope="module")
def built():
    from recallable_kv_cache_cosine_b200 import build
    build.build()
    return ckv.lib()


def test_header_declares_the_three_entry_points():
    names = _declared_functions()
    for n in ("cluster_prefill", "select_and_attend", "recluster_increment"):
        assert n in names


def test_library_exports_every_declared_symbol(built):
    names = _declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", ckv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared in ckv.h but not exported: {missing}"
    # nothing but the ABI is exported (hidden visibility for everything else)
    extra = sorted(e for e in exported if e not in set(names))
    assert not extra, f"unexpected exports: {extra}"
    assert set(ckv.SIGNATURES) == set(names)


def test_config_defaults_and_error_strings(built):
    cfg = ckv.Config()
    assert built.ckv_config_default(C.byref(cfg)) == 0
    assert (cfg.n_sink, cfg.window, cfg.new_clusters, cfg.iters, cfg.head_dim) == (16, 320, 4, 10, 128)
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert built.ckv_strerror(code)
    assert built.ckv_config_default(None) == ckv.CKV_EINVAL


def test_create_rejects_bad_config_before_touching_the_device(built):
    cfg = ckv.Config()
    built.ckv_config_default(C.byref(cfg))
    ctx = C.c_void_p()
    cfg.head_dim = 64
    assert built.ckv_create(C.byref(cfg), C.byref(ctx)) == ckv.CKV_EINVAL
    assert b"head_dim" in built.ckv_last_error()
    built.ckv_config_default(C.byref(cfg))
    cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.n_q_heads = 1, 1, 8, 12
    cfg.capacity, cfg.max_clusters = 1024, 64
    assert built.ckv_create(C.byref(cfg), C.byref(ctx)) == ckv.CKV_EINVAL  # 12 % 8 != 0
    cfg.n_q_heads = 128
    assert built.ckv_create(C.byref(cfg), C.byref(ctx)) == ckv.CKV_EINVAL  # group 16 > 8
    cfg.n_q_heads, cfg.max_clusters = 32, 5000
    assert built.ckv_create(C.byref(cfg), C.byref(ctx)) == ckv.CKV_EINVAL
    assert built.ckv_create(None, C.byref(ctx)) == ckv.CKV_EINVAL


def test_calls_on_null_context_fail_cleanly(built):
    assert built.cluster_prefill(None, 0, None, None, 100, 4, None) == ckv.CKV_EINVAL
    assert built.select_and_attend(None, 0, None, 64, None, None, None, None) == ckv.CKV_EINVAL
    assert built.recluster_increment(None, 0, None) == ckv.CKV_EINVAL
    assert built.ckv_destroy(None) == 0


def test_every_context_call_rejects_a_null_context(built):
    """Each entry point that takes a context checks it on the host first: a null context is
    CKV_EINVAL, with no device call."""
    no_ctx = {"ckv_config_default", "ckv_create", "ckv_destroy", "ckv_strerror",
              "ckv_last_error", "ckv_device_bytes", "ckv_kmeans_update_noalloc"}
    checked = []
    for name, (_, argtypes) in ckv.SIGNATURES.items():
        if name in no_ctx:
            continue
        args = [None] + [0.0 if t is C.c_float else (None if t is C.c_void_p else 0)
                         for t in argtypes[1:]]
        assert getattr(built, name)(*args) == ckv.CKV_EINVAL, name
        assert built.ckv_last_error(), name
        checked.append(name)
    assert "split_drifted_clusters" in checked and "select_and_attend_per_head" in checked
    assert built.ckv_device_bytes(None) == 0


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "recallable_kv_cache_cosine_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "ckv_oracle" not in txt and "libckv_oracle" not in txt, f


def test_binding_constants_and_structs_match_the_header():
    src = open(HEADER).read()
    codes = dict(re.findall(r"#define (CKV_E\w+|CKV_OK)\s+\(?(-?\d+)\)?", src))
    assert codes and all(getattr(ckv, k) == int(v) for k, v in codes.items()), codes
    # field order and types of the structs the binding mirrors
    for cname, pyt in (("ckv_config", ckv.Config), ("ckv_layer_info", ckv.LayerInfo),
                       ("ckv_unit_buffers", ckv.UnitBuffers)):
        body = re.search(r"typedef struct %s \{(.*?)\} %s;" % (cname, cname), src, re.S).group(1)
        body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
        decls = re.findall(r"([\w ]+?)\s*(\*?)\s*(\w+)\s*;", body)
        assert [d[2] for d in decls] == [f for f, _ in pyt._fields_], (cname, decls)
        ctype = {"int32_t": C.c_int32, "int64_t": C.c_int64, "uint64_t": C.c_uint64}
        for (typ, star, name), (_, pt) in zip(decls, pyt._fields_):
            want = C.c_void_p if star else ctype[typ.strip()]
            assert pt is want, (cname, name, typ, star, pt)
