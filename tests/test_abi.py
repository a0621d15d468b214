"""The C ABI without a GPU: the library loads, exports every entry point include/ekv.h
declares, its struct layout matches the binding's, and host-side validation answers with the
documented status codes before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ekv.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_kv_cache_kmin_b200 import build, ekv
    build.build_library()
    return ekv.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(ekv_[a-z_0-9]+)\s*\(",
                                 text, re.M)))


def test_header_declares_the_four_calls_and_helpers():
    names = declared_functions()
    for n in ["ekv_page_meta_update", "ekv_score_pages", "ekv_select_pages", "ekv_sparse_decode",
              "ekv_decode_workspace_bytes", "ekv_device_status", "ekv_clear_device_status",
              "ekv_status_str"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from sparse_kv_cache_kmin_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ekv_\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert hasattr(lib, n)


def test_struct_layout_matches_header(tmp_path):
    from sparse_kv_cache_kmin_b200.ekv import EkvCacheStruct
    src = tmp_path / "layout.c"
    fields = [f for f, _ in EkvCacheStruct._fields_]
    body = "".join('printf("%%s %%zu\\n", "%s", offsetof(ekv_cache, %s));' % (f, f) for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "ekv.h"\nint main(void){%s'
                   'printf("sizeof %%zu\\n", sizeof(ekv_cache));return 0;}\n' % body)
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())
    for f in fields:
        assert int(got[f]) == getattr(EkvCacheStruct, f).offset, f
    assert int(got["sizeof"]) == ctypes.sizeof(EkvCacheStruct)


def test_status_strings(lib):
    from sparse_kv_cache_kmin_b200 import ekv
    assert lib.ekv_status_str(ekv.EKV_OK) == b"EKV_OK"
    assert lib.ekv_status_str(ekv.EKV_ERR_WORKSPACE) == b"EKV_ERR_WORKSPACE"
    assert lib.ekv_status_str(99) == b"EKV_UNKNOWN_STATUS"


def fake_cache(**over):
    """A struct with non-null placeholder pointers: host validation only reads sizes and
    checks pointers for NULL, so no device memory is touched by the failing calls below."""
    from sparse_kv_cache_kmin_b200.ekv import EkvCacheStruct
    c = EkvCacheStruct()
    c.dtype, c.head_dim, c.page_size, c.num_kv_heads = 1, 128, 16, 8
    c.num_blocks, c.batch, c.max_pages, c.reserved = 1024, 4, 256, 0
    for f in ["k_cache", "v_cache", "meta_bbox", "meta_mom", "page_table", "seq_lens", "dev_status"]:
        setattr(c, f, 0x1000)
    for k, v in over.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("over,status", [
    ({"head_dim": 96}, 2), ({"page_size": 8}, 2), ({"dtype": 7}, 2),
    ({"num_kv_heads": 0}, 1), ({"k_cache": None}, 1), ({"dev_status": None}, 1),
    ({"batch": 9000}, 2), ({"meta_bbox": 0x1008}, 1),
])
def test_score_validation(lib, over, status):
    c = fake_cache(**over)
    assert lib.ekv_score_pages(ctypes.byref(c), 0x1000, 32, 1.0, 0, 0x1000, None) == status


def test_head_count_and_policy_validation(lib):
    c = fake_cache()
    assert lib.ekv_score_pages(ctypes.byref(c), 0x1000, 30, 1.0, 0, 0x1000, None) == 1   # H_q % H_kv
    assert lib.ekv_score_pages(ctypes.byref(c), 0x1000, 8 * 16, 1.0, 0, 0x1000, None) == 2  # G = 16
    assert lib.ekv_score_pages(ctypes.byref(c), 0x1000, 32, 0.0, 0, 0x1000, None) == 1   # scale
    assert lib.ekv_score_pages(ctypes.byref(c), 0x1000, 32, 1.0, 5, 0x1000, None) == 2   # policy
    c2 = fake_cache(meta_mom=None)
    assert lib.ekv_score_pages(ctypes.byref(c2), 0x1000, 32, 1.0, 1, 0x1000, None) == 1  # gauss w/o moments
    c3 = fake_cache(meta_mom=0x1004)
    assert lib.ekv_score_pages(ctypes.byref(c3), 0x1000, 32, 1.0, 1, 0x1000, None) == 1  # misaligned moments


def test_select_validation(lib):
    c = fake_cache()
    P = 0x1000
    assert lib.ekv_select_pages(ctypes.byref(c), 32, 0, 0, 1.5, 0.1, P, P, P, 16, None, None) == 1
    assert lib.ekv_select_pages(ctypes.byref(c), 32, 0, 64, 1.5, 0.1, P, P, P, 16, None, None) == 1
    assert lib.ekv_select_pages(ctypes.byref(c), 32, 1, 0, 1.2, 0.1, P, P, P, 16, P, None) == 2
    assert lib.ekv_select_pages(ctypes.byref(c), 32, 1, 0, 1.5, 0.1, P, P, P, 16, None, None) == 1


def test_decode_validation_and_workspace(lib):
    c = fake_cache()
    P = 0x1000
    need = lib.ekv_decode_workspace_bytes(ctypes.byref(c), 32, 256)
    assert need > 0
    # [B*H_q][NC][2] + [B*H_q][NC][D] + [B*H_q][NC*CP*P] floats + [B*H_kv][max_sel] ints,
    # each 256-byte aligned
    assert need >= 4 * 32 * 256 * 16 * 4 + 4 * 8 * 256 * 4
    assert lib.ekv_decode_workspace_bytes(ctypes.byref(c), 30, 256) == 0
    assert lib.ekv_sparse_decode(ctypes.byref(c), P, 32, 1.0, 1, P, P, 256, P, P, P, need - 1, None) == 3
    assert lib.ekv_sparse_decode(ctypes.byref(c), P, 32, 1.0, 1, P, P, 256, P, P, None, need, None) == 3
    assert lib.ekv_sparse_decode(ctypes.byref(c), P, 32, 1.0, 9, P, P, 256, P, P, P, need, None) == 2
    c2 = fake_cache(v_cache=None)
    assert lib.ekv_sparse_decode(ctypes.byref(c2), P, 32, 1.0, 1, P, P, 256, P, P, P, need, None) == 1


def test_meta_update_validation(lib):
    c = fake_cache()
    assert lib.ekv_page_meta_update(ctypes.byref(c), None, 0x1000, 16, None) == 1
    assert lib.ekv_page_meta_update(ctypes.byref(c), 0x1000, 0x1000, -1, None) == 1
    assert lib.ekv_page_meta_update(ctypes.byref(c), 0x1000, 0x1000, 256 * 16 + 1, None) == 1


def test_binding_refuses_host_tensors():
    import torch
    from sparse_kv_cache_kmin_b200 import ekv
    with pytest.raises(ValueError):
        ekv._ptr(torch.zeros(4))


def test_product_path_does_not_import_the_oracle():
    # The package must not reach the CPU oracle: no import of it anywhere in the product.
    pkg = os.path.join(ROOT, "sparse_kv_cache_kmin_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
                assert "ekv_oracle" not in text, f


def test_moment_entry_points_validation(lib):
    from sparse_kv_cache_kmin_b200.ekv import load_library
    import ctypes as C
    P = 0x1000
    lib = load_library()
    cp = C.POINTER(type(fake_cache()))
    lib.ekv_moment_bytes.argtypes, lib.ekv_moment_bytes.restype = [cp], C.c_size_t
    lib.ekv_moment_decode_workspace_bytes.argtypes = [cp, C.c_int32, C.c_int32]
    lib.ekv_moment_decode_workspace_bytes.restype = C.c_size_t
    lib.ekv_moment_update.argtypes = [cp, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p]
    lib.ekv_sparse_decode_moment.argtypes = [cp, C.c_void_p, C.c_void_p, C.c_int32, C.c_float,
                                             C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p,
                                             C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
    c = fake_cache()
    # [batch][H_kv] records of 4 + 2d + d*d floats
    assert lib.ekv_moment_bytes(C.byref(c)) == 4 * 8 * (4 + 2 * 128 + 128 * 128) * 4
    assert lib.ekv_moment_bytes(C.byref(fake_cache(v_cache=None))) == 0
    base = lib.ekv_decode_workspace_bytes(C.byref(c), 32, 256)
    need = lib.ekv_moment_decode_workspace_bytes(C.byref(c), 32, 256)
    # the decode workspace, then [batch][H_kv] records of 4 + 2d + G*d floats
    assert need >= base + 4 * 8 * (4 + 2 * 128 + 4 * 128) * 4
    assert lib.ekv_moment_decode_workspace_bytes(C.byref(c), 30, 256) == 0
    assert lib.ekv_moment_update(C.byref(c), None, P, P, 16, None) == 1
    assert lib.ekv_moment_update(C.byref(c), P, P, P, -1, None) == 1
    assert lib.ekv_moment_update(C.byref(c), P, P, P, 256 * 16 + 1, None) == 1
    assert lib.ekv_sparse_decode_moment(C.byref(c), None, P, 32, 1.0, P, P, 256, P, P, P, need, None) == 1
    assert lib.ekv_sparse_decode_moment(C.byref(c), P, P, 32, 1.0, P, P, 256, P, P, P, need - 1, None) == 3
    assert lib.ekv_sparse_decode_moment(C.byref(c), P, P, 30, 1.0, P, P, 256, P, P, P, need, None) == 1
    assert lib.ekv_sparse_decode_moment(C.byref(c), P, P, 32, 0.0, P, P, 256, P, P, P, need, None) == 1


def test_token_entry_points_validation(lib):
    from sparse_kv_cache_kmin_b200.ekv import load_library
    import ctypes as C
    P = 0x1000
    lib = load_library()
    cp = C.POINTER(type(fake_cache()))
    vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
    lib.ekv_token_workspace_bytes.argtypes = [cp, i32]
    lib.ekv_token_workspace_bytes.restype = C.c_size_t
    lib.ekv_select_tokens.argtypes = [cp, vp, i32, f32, vp, vp, i32, i32, vp, vp, vp, vp, C.c_size_t, vp]
    lib.ekv_sparse_decode_tokens.argtypes = [cp, vp, i32, f32, i32, vp, vp, vp, i32, vp, vp, vp]
    c = fake_cache()
    need = lib.ekv_token_workspace_bytes(C.byref(c), 256)
    assert need == 4 * 8 * 256 * 16 * 4  # one fp32 score per candidate slot
    assert lib.ekv_token_workspace_bytes(C.byref(c), 0) == 0
    sel = lambda T, ws=need: lib.ekv_select_tokens(C.byref(c), P, 32, 1.0, P, P, 256, T, P, P, P, P, ws, None)
    assert sel(0) == 1
    assert sel(32769) == 2
    assert sel(512, need - 1) == 3
    dec = lambda attn, T: lib.ekv_sparse_decode_tokens(C.byref(c), P, 32, 1.0, attn, P, P, P, T, P, P, None)
    assert dec(7, 64) == 2
    assert dec(1, 0) == 1
    assert dec(1, 32769) == 2
    c2 = fake_cache(v_cache=None)
    assert lib.ekv_sparse_decode_tokens(C.byref(c2), P, 32, 1.0, 1, P, P, P, 64, P, P, None) == 1


def test_misaligned_scores_and_workspaces_are_refused_before_any_launch(lib):
    # select reads score rows as float4 and the decode reads logits back from its workspace as
    # float4: a pointer 4 or 8 bytes off a 16-byte boundary (a tensor slice, say) is refused on
    # the host with EKV_ERR_INVALID_ARG; the placeholder pointers are never dereferenced
    import ctypes as C
    from sparse_kv_cache_kmin_b200.ekv import load_library
    lib = load_library()
    cp = C.POINTER(type(fake_cache()))
    vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
    c = fake_cache()
    P = 0x1000
    for off in (4, 8):
        assert lib.ekv_select_pages(C.byref(c), 32, 0, 64, 1.5, 0.1, P + off, P, P, 64, None, None) == 1
        assert lib.ekv_select_pages(C.byref(c), 32, 1, 0, 1.5, 0.1, P + off, P, P, 64, P, None) == 1
    need = lib.ekv_decode_workspace_bytes(C.byref(c), 32, 256)
    for off in (4, 8):
        assert lib.ekv_sparse_decode(C.byref(c), P, 32, 1.0, 1, P, P, 256, P, P, P + off, need + 16,
                                     None) == 1
    lib.ekv_moment_decode_workspace_bytes.argtypes = [cp, i32, i32]
    lib.ekv_moment_decode_workspace_bytes.restype = C.c_size_t
    lib.ekv_sparse_decode_moment.argtypes = [cp, vp, vp, i32, f32, vp, vp, i32, vp, vp, vp,
                                             C.c_size_t, vp]
    mneed = lib.ekv_moment_decode_workspace_bytes(C.byref(c), 32, 256)
    assert lib.ekv_sparse_decode_moment(C.byref(c), P, P, 32, 1.0, P, P, 256, P, P, P + 4,
                                        mneed + 16, None) == 1
    lib.ekv_token_workspace_bytes.argtypes = [cp, i32]
    lib.ekv_token_workspace_bytes.restype = C.c_size_t
    lib.ekv_select_tokens.argtypes = [cp, vp, i32, f32, vp, vp, i32, i32, vp, vp, vp, vp,
                                      C.c_size_t, vp]
    tneed = lib.ekv_token_workspace_bytes(C.byref(c), 256)
    assert lib.ekv_select_tokens(C.byref(c), P, 32, 1.0, P, P, 256, 512, P, P, P, P + 8,
                                 tneed + 16, None) == 1


def test_select_decode_validation(lib):
    # the one-call selection + decode refuses what either of its halves refuses, on the host
    import ctypes as C
    cp = C.POINTER(type(fake_cache()))
    vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
    fn = lib.ekv_select_decode
    fn.argtypes = [cp, vp, i32, f32, i32, i32, vp, vp, vp, i32, vp, vp, vp, C.c_size_t, vp]
    c = fake_cache()
    P = 0x1000
    need = lib.ekv_decode_workspace_bytes(C.byref(c), 32, 256)

    def call(topk=64, scores=P, max_sel=256, attn=1, ws=P, ws_bytes=None, q=P, cache=c):
        return fn(C.byref(cache), q, 32, 1.0, attn, topk, scores, P, P, max_sel, P, P, ws,
                  need if ws_bytes is None else ws_bytes, None)

    assert call(topk=0) == 1                      # k < 1
    assert call(topk=200, max_sel=100) == 1       # max_sel < min(k, max_pages)
    assert call(scores=None) == 1
    assert call(scores=P + 4) == 1                # score rows are read as float4
    assert call(q=P + 8) == 1                     # query rows move with 16-byte loads
    assert call(attn=9) == 2
    assert call(ws_bytes=need - 1) == 3
    assert call(ws=None) == 3
    assert call(ws=P + 4, ws_bytes=need + 16) == 1
    assert call(cache=fake_cache(v_cache=None)) == 1


def test_wait_selftest_validation(lib):
    import ctypes as C
    cp = C.POINTER(type(fake_cache()))
    lib.ekv_wait_selftest.argtypes = [cp, C.c_uint64, C.c_void_p]
    c = fake_cache()
    assert lib.ekv_wait_selftest(C.byref(c), 2_000_000_001, None) == 1   # above the 2 s limit
    c2 = fake_cache(dev_status=None)
    assert lib.ekv_wait_selftest(C.byref(c2), 1000, None) == 1


def test_refresh_score_validation(lib):
    # the one-call metadata refresh + scores refuses what either of its halves refuses, on the
    # host; every call below fails validation, so nothing is launched
    import ctypes as C
    cp = C.POINTER(type(fake_cache()))
    vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
    fn = lib.ekv_refresh_score_pages
    fn.argtypes = [cp, vp, vp, i32, vp, i32, f32, i32, vp, vp]
    P = 0x1000

    def call(start=P, count=P, max_new=16, q=P, hq=32, scale=1.0, policy=0, scores=P, cache=None):
        c = fake_cache() if cache is None else cache
        return fn(C.byref(c), start, count, max_new, q, hq, scale, policy, scores, None)

    assert call(start=None) == 1
    assert call(count=None) == 1
    assert call(max_new=-1) == 1
    assert call(max_new=256 * 16 + 1) == 1        # longer than a whole sequence
    assert call(cache=fake_cache(k_cache=P + 4)) == 1
    assert call(q=None) == 1
    assert call(scores=None) == 1
    assert call(scale=0.0) == 1
    assert call(scale=float("inf")) == 1
    assert call(hq=31) == 1                       # not a multiple of H_kv
    assert call(hq=8 * 16) == 2                   # G = 16
    assert call(policy=7) == 2
    assert call(policy=1, cache=fake_cache(meta_mom=None)) == 1
    assert call(cache=fake_cache(meta_bbox=P + 8)) == 1
    assert call(policy=2, cache=fake_cache(meta_mom=P + 4)) == 1
    assert call(cache=fake_cache(dtype=5)) == 2
