"""Host-side checks of the C ABI (no GPU needed, nothing is launched):
libcsa.so loads, exports every function include/csa.h declares, sizes its
workspaces, and rejects bad arguments before any launch."""
import ctypes as C
import os
import re

import pytest

from long_context_sparse_09_b200 import binding as bd
from long_context_sparse_09_b200.configs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "csa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:csa|hca)_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(bd.LIB_PATH):
        from long_context_sparse_09_b200 import build
        build.build_library()
    return bd.lib()


def test_header_declares_the_four_calls():
    names = _declared()
    for n in ("csa_compress", "hca_compress", "csa_index_topk", "csa_attend", "hca_attend"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(bd.exported_symbols())
    assert lib.csa_abi_version() == 1


def test_nm_lists_the_symbols(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True,
                         text=True).stdout
    for name in _declared():
        assert re.search(rf"\sT\s{name}$", out, re.M), name


def test_workspace_sizes(lib):
    wl = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(wl)
    N = wl.T // wl.m
    assert lib.csa_index_topk_workspace_bytes(C.byref(p), 4, 1, N) >= 4 * N * 4
    assert lib.csa_attend_workspace_bytes(C.byref(p), 4, 1, N) > 0
    w3 = WORKLOADS["flash_csa_prefill_32k"]
    p3 = bd.params_for(w3)
    assert lib.csa_compress_workspace_bytes(C.byref(p3), 1, 4096, w3.d) >= 4096 * (4 * 512 + 4 * 128) * 4
    assert lib.csa_packed_weight_bytes(C.byref(p3), w3.d) >= (4 * 512 + 4 * 128) * w3.d * 2


def test_status_strings(lib):
    for s in range(9):
        assert lib.csa_status_string(s)


def test_argument_errors_return_before_launch(lib):
    wl = WORKLOADS["flash_csa_decode_64k"]
    p = bd.params_for(wl)
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    # null query positions
    st = lib.csa_index_topk(C.byref(p), 1, 1, None, fake, fake, fake, 16, fake, None, fake,
                            1 << 30, None)
    assert st == 1  # CSA_ERR_ARG
    # bad shape
    st = lib.csa_index_topk(C.byref(p), 0, 1, fake, fake, fake, fake, 16, fake, None, fake,
                            1 << 30, None)
    assert st == 2
    # misaligned pointer
    st = lib.csa_index_topk(C.byref(p), 1, 1, fake, C.c_void_p((1 << 20) + 2), fake, fake, 16,
                            fake, None, fake, 1 << 30, None)
    assert st == 3
    # workspace too small
    st = lib.csa_index_topk(C.byref(p), 1, 1, fake, fake, fake, fake, 16, fake, None, fake,
                            4, None)
    assert st == 8
    # wrong variant for the call
    ph = bd.params_for(WORKLOADS["hca_decode_1m"])
    st = lib.csa_attend(C.byref(ph), 1, 1, fake, fake, fake, fake, None, 16, fake, None, 128,
                        fake, fake, fake, fake, 1 << 30, None)
    assert st == 1
    # FP8-mixed cache without its scale plane
    p4 = bd.params_for(WORKLOADS["pro_csa_decode_1m"])
    st = lib.csa_attend(C.byref(p4), 1, 1, fake, fake, fake, fake, None, 16, fake, fake, 128,
                        fake, fake, fake, fake, 1 << 30, None)
    assert st == 1
    # unsupported dtype
    bad = bd.params_for(wl)
    bad.act = 7
    st = lib.csa_attend(C.byref(bad), 1, 1, fake, fake, fake, fake, None, 16, fake, None, 128,
                        fake, fake, fake, fake, 1 << 30, None)
    assert st == 4


def test_decode_append_argument_errors(lib):
    wl = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(wl)
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    d = wl.d
    # per sequence: C^a of the last token, then two slots of (max, den, num) per channel
    assert lib.csa_decode_tail_bytes(C.byref(p), 4, d) == 4 * (wl.c + 2 * 3 * (wl.c + wl.c_I)) * 4
    # indexer keys missing for the CSA variant
    st = lib.csa_decode_append(C.byref(p), 4, d, fake, fake, fake, fake, fake, fake, 16, None,
                               None, None, None, 0, None)
    assert st == 1
    # d not a multiple of 8 bf16 elements
    st = lib.csa_decode_append(C.byref(p), 4, d + 4, fake, fake, fake, fake, fake, fake, 16, fake,
                               None, None, None, 0, None)
    assert st == 2
    # the HCA call with CSA parameters
    st = lib.hca_decode_append(C.byref(p), 4, d, fake, fake, fake, fake, fake, fake, 16, None,
                               None, None, 0, None)
    assert st == 1
    # a window without its base positions
    ph = bd.params_for(WORKLOADS["hca_decode_1m"])
    st = lib.hca_decode_append(C.byref(ph), 2, wl.d, fake, fake, fake, fake, fake, None, 16, fake,
                               None, None, 128, None)
    assert st == 1


def test_out_proj_sizes_and_argument_errors(lib):
    # V4-Pro: c = 512, n_h = 128, g = 16, d_g = 1024, d = 7168
    assert lib.csa_out_proj_packed_bytes(128, 512, 16, 1024, 7168) == \
        16 * 1024 * 4096 * 2 + 7168 * 16384 * 2
    assert lib.csa_out_proj_workspace_bytes(4, 128, 512, 16, 1024, 7168) == 4 * 16384 * 2
    # unsupported shapes: heads not divisible into groups, c n_h / g not a
    # multiple of 64, d_g not a multiple of 128
    assert lib.csa_out_proj_packed_bytes(128, 512, 12, 1024, 7168) == 0
    assert lib.csa_out_proj_packed_bytes(8, 4, 2, 128, 64) == 0
    assert lib.csa_out_proj_packed_bytes(8, 64, 2, 100, 64) == 0
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = 1 << 30
    assert lib.csa_out_proj(4, 128, 512, 12, 1024, 7168, fake, fake, fake, fake, ws, None) == 2
    assert lib.csa_out_proj(0, 128, 512, 16, 1024, 7168, fake, fake, fake, fake, ws, None) == 2
    assert lib.csa_out_proj(4, 128, 512, 16, 1024, 7168, None, fake, fake, fake, ws, None) == 1
    assert lib.csa_out_proj(4, 128, 512, 16, 1024, 7168, C.c_void_p((1 << 20) + 8), fake, fake,
                            fake, ws, None) == 3
    assert lib.csa_out_proj(4, 128, 512, 16, 1024, 7168, fake, fake, fake, None, 0, None) == 8
    assert lib.csa_out_proj(4, 128, 512, 16, 1024, 7168, fake, fake, fake, fake, 16, None) == 8
    assert lib.csa_out_proj_pack(128, 512, 16, 1024, 7168, None, fake, fake, None) == 1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(bd, "_lib", None)
    monkeypatch.setattr(bd, "LIB_PATH", str(tmp_path / "libcsa.so"))
    with pytest.raises(RuntimeError):
        bd.lib()


def test_binding_checks_dtypes_and_sizes_before_the_call(lib):
    import torch
    O = torch.zeros(2, 8, 64)  # fp32: the call reads bf16
    out = torch.zeros(2, 200, dtype=torch.bfloat16)
    packed = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="O"):
        bd.csa_out_proj(O, packed, 2, 128, out)
    with pytest.raises(ValueError, match="packed"):  # smaller than the packed weights
        bd.csa_out_proj(O.to(torch.bfloat16), packed, 2, 128, out)
    with pytest.raises(ValueError, match="WG"):
        bd.out_proj_pack(torch.zeros(2, 256, 128), torch.zeros(256, 200, dtype=torch.bfloat16))


def test_binding_checks_decode_append_inputs(lib):
    import torch
    wl = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(wl)
    B, d = 2, wl.d
    H = torch.zeros(B, d)  # fp32 for a bf16 configuration
    t = torch.zeros(B, dtype=torch.int32)
    tail = torch.zeros(bd.decode_tail_bytes(p, B, d) // 4)
    with pytest.raises(ValueError, match="H"):
        bd.csa_decode_append(p, H, t, None, tail, None, None, None, None, None, None)
    with pytest.raises(ValueError, match="tail"):
        bd.csa_decode_append(p, H.to(torch.bfloat16), t, None, tail[:10], None, None, None,
                             None, None, None)
    with pytest.raises(ValueError, match="t"):
        bd.hca_decode_append(bd.params_for(WORKLOADS["hca_decode_1m"]),
                             torch.zeros(B, 4096, dtype=torch.bfloat16), t.long(), None, tail,
                             None, None, None, None, None)
