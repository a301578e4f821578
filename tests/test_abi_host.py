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
    with pytest.raises(ValueError, match=r"^O:"):
        bd.csa_out_proj(O, packed, 2, 128, out)
    with pytest.raises(ValueError, match=r"^packed:"):  # smaller than the packed weights
        bd.csa_out_proj(O.to(torch.bfloat16), packed, 2, 128, out)
    with pytest.raises(ValueError, match=r"^WG:"):
        bd.out_proj_pack(torch.zeros(2, 256, 128), torch.zeros(256, 200, dtype=torch.bfloat16))


def test_binding_checks_decode_append_inputs(lib):
    import torch
    wl = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(wl)
    B, d = 2, wl.d
    H = torch.zeros(B, d)  # fp32 for a bf16 configuration
    t = torch.zeros(B, dtype=torch.int32)
    tail = torch.zeros(bd.decode_tail_bytes(p, B, d) // 4)
    with pytest.raises(ValueError, match=r"^H:"):
        bd.csa_decode_append(p, H, t, None, tail, None, None, None, None, None, None)
    with pytest.raises(ValueError, match=r"^tail:"):
        bd.csa_decode_append(p, H.to(torch.bfloat16), t, None, tail[:10], None, None, None,
                             None, None, None)
    ph = bd.params_for(WORKLOADS["hca_decode_1m"])
    tail_h = torch.zeros(bd.decode_tail_bytes(ph, B, 4096) // 4)  # right size: only t is wrong
    with pytest.raises(ValueError, match=r"^t:"):
        bd.hca_decode_append(ph, torch.zeros(B, 4096, dtype=torch.bfloat16), t.long(), None,
                             tail_h, None, None, None, None, None)


def _index_tensors(p, B=2, Q=3, N=40):
    import torch
    adt = torch.bfloat16
    R = B * Q
    return dict(q_pos=torch.zeros(R, dtype=torch.int32),
                qI=torch.zeros(R, p.n_hI, p.c_I, dtype=adt),
                w=torch.zeros(R, p.n_hI),
                kI=torch.zeros(B, N, p.c_I, dtype=adt),
                idx_out=torch.zeros(R, p.topk, dtype=torch.int32),
                score_out=torch.zeros(R, p.topk))


@pytest.mark.parametrize("fn", ["csa_index_topk", "csa_index_topk_noalloc"])
@pytest.mark.parametrize("bad,what", [
    (dict(idx_out=("shape", (6, 10))), r"^idx_out:"),
    (dict(idx_out=("dtype", "int64")), r"^idx_out:"),
    (dict(score_out=("shape", (6, 10))), r"^score_out:"),
    (dict(q_pos=("dtype", "int64")), r"^q_pos:"),
    (dict(q_pos=("shape", (2,))), r"^q_pos:"),
    (dict(w=("dtype", "bfloat16")), r"^w:"),
    (dict(qI=("dtype", "float32")), r"^qI:"),
    (dict(kI=("shape", (2, 40, 64))), r"^kI:"),
])
def test_binding_checks_index_topk_tensors(lib, fn, bad, what):
    """Every tensor csa_index_topk reads or writes is checked for its dtype
    and size before the call (an undersized output would be written past
    its end on the device)."""
    import torch
    p = bd.params_for(WORKLOADS["flash_csa_decode_64k"])
    t = _index_tensors(p)
    for k, (kind, v) in bad.items():
        t[k] = (torch.zeros(v, dtype=t[k].dtype) if kind == "shape"
                else t[k].to(getattr(torch, v)))
    f = getattr(bd, fn)
    with pytest.raises(ValueError, match=what):
        f(p, t["q_pos"], t["qI"], t["w"], t["kI"], t["idx_out"], t["score_out"])


def test_binding_rejects_queries_not_divisible_by_sequences(lib):
    import torch
    p = bd.params_for(WORKLOADS["flash_csa_decode_64k"])
    t = _index_tensors(p, B=2, Q=3)
    t["kI"] = torch.zeros(4, 40, p.c_I, dtype=torch.bfloat16)  # 6 query rows, 4 sequences
    with pytest.raises(ValueError, match=r"^qI:.*whole number"):
        bd.csa_index_topk(p, t["q_pos"], t["qI"], t["w"], t["kI"], t["idx_out"])


def _attend_tensors(wl, B=2, Q=1, N=50, W=128):
    import torch
    from long_context_sparse_09_b200 import synth
    R = B * Q
    st = synth._Streams(0, "cpu")
    ckv, ckv_s = synth.cache_rows(wl, st, "ckv", (B,), N)
    win, win_s = synth.cache_rows(wl, st, "win", (B,), W)
    return dict(q_pos=torch.zeros(R, dtype=torch.int32),
                q=torch.zeros(R, wl.n_h, wl.c, dtype=torch.bfloat16),
                idx=torch.zeros(R, wl.topk, dtype=torch.int32),
                ckv=ckv, ckv_scale=ckv_s, win=win, win_scale=win_s,
                win_pos0=torch.zeros(B, dtype=torch.int32),
                sink=torch.zeros(wl.n_h),
                out=torch.zeros(R, wl.n_h, wl.c, dtype=torch.bfloat16))


@pytest.mark.parametrize("wname", ["pro_csa_decode_1m", "hca_decode_1m"])
@pytest.mark.parametrize("key,repl,what", [
    ("out", lambda t: t[:1], r"^out:"),
    ("out", lambda t: t.float(), r"^out:"),
    ("q", lambda t: t.float(), r"^q:"),
    ("q_pos", lambda t: t.long(), r"^q_pos:"),
    ("sink", lambda t: t[:3], r"^sink:"),
    ("idx", lambda t: t[:, :5].contiguous(), r"^idx:"),
    ("ckv", lambda t: t[..., :100].contiguous(), r"^ckv:"),  # rows too short
    ("ckv_scale", lambda t: None if t is None else t[:, :10].contiguous(), r"^ckv_scale:"),
    ("win", lambda t: t.view(-1)[:100].view(1, 1, 100), r"^win"),
    ("win_pos0", lambda t: t[:1], r"^win_pos0:"),
])
def test_binding_checks_attend_tensors(lib, wname, key, repl, what):
    """Every tensor csa_attend / hca_attend reads or writes is checked for
    its dtype and size before the call, the KV caches in their format (FP8
    records in uint8 with their scale plane)."""
    wl = WORKLOADS[wname]
    t = _attend_tensors(wl)
    if key == "idx" and wl.variant == "hca":
        pytest.skip("hca_attend takes no selection")
    if key == "ckv_scale" and wl.kv != "fp8mix":
        t["ckv_scale"] = t["ckv"][:, :, 0].float()  # a scale plane for a bf16 cache
    else:
        t[key] = repl(t[key])
    p = bd.params_for(wl)
    with pytest.raises(ValueError, match=what):
        if wl.variant == "csa":
            bd.csa_attend(p, t["q_pos"], t["q"], t["idx"], t["ckv"], t["ckv_scale"], t["win"],
                          t["win_scale"], t["win_pos0"], t["sink"], t["out"])
        else:
            bd.hca_attend(p, t["q_pos"], t["q"], t["ckv"], t["ckv_scale"], t["win"],
                          t["win_scale"], t["win_pos0"], t["sink"], t["out"])


def test_binding_checks_compress_tensors(lib):
    import torch
    wl = WORKLOADS["tiny_csa_prefill_f32"].with_(act="bf16", kv="fp8mix")
    p = bd.params_for(wl)
    B, T = 1, 64
    nE = T // wl.m
    H = torch.zeros(B, T, wl.d, dtype=torch.bfloat16)
    packed = torch.zeros(lib.csa_packed_weight_bytes(C.byref(p), wl.d), dtype=torch.uint8)
    rb = bd.kv_row_bytes(p)
    ckv = torch.zeros(B, nE, rb, dtype=torch.uint8)
    ckv_s = torch.zeros(B, nE)
    kI = torch.zeros(B, nE, wl.c_I, dtype=torch.bfloat16)
    win = torch.zeros(B, T, rb, dtype=torch.uint8)
    win_s = torch.zeros(B, T)
    with pytest.raises(ValueError, match=r"^H:"):
        bd.csa_compress(p, H.float(), packed, ckv, ckv_s, kI, win, win_s)
    with pytest.raises(ValueError, match=r"^packed:"):
        bd.csa_compress(p, H, packed[:100], ckv, ckv_s, kI, win, win_s)
    with pytest.raises(ValueError, match=r"^ckv:"):
        bd.csa_compress(p, H, packed, ckv[:, :3], ckv_s, kI, win, win_s)
    with pytest.raises(ValueError, match=r"^ckv_scale:"):
        bd.csa_compress(p, H, packed, ckv, None, kI, win, win_s)
    with pytest.raises(ValueError, match=r"^kI:"):
        bd.csa_compress(p, H, packed, ckv, ckv_s, kI.float(), win, win_s)
    with pytest.raises(ValueError, match=r"^win_scale:"):
        bd.csa_compress(p, H, packed, ckv, ckv_s, kI, win, win_s[:, :5])


def test_noalloc_scratch_bound_is_the_workspace_size(lib):
    """csa_index_topk_noalloc accepts exactly the requests whose
    csa_index_topk workspace is at most its 16 MiB scratch: just below the
    boundary it passes the size check (and stops at the null query
    positions, or at the device lookup on a host without a GPU, before any
    launch); just above it returns CSA_ERR_WORKSPACE."""
    p = bd.params_for(WORKLOADS["pro_csa_decode_1m"])
    cap = 16 << 20
    ws = lambda n: lib.csa_index_topk_workspace_bytes(C.byref(p), 4, 1, n)
    lo, hi = 1, 1 << 22  # ws(lo) <= cap < ws(hi)
    assert ws(lo) <= cap < ws(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if ws(mid) <= cap:
            lo = mid
        else:
            hi = mid
    fake = C.c_void_p(1 << 20)  # never dereferenced: checks come first
    st_lo = lib.csa_index_topk_noalloc(C.byref(p), 4, 1, None, fake, fake, fake, lo, fake,
                                       None, None)
    st_hi = lib.csa_index_topk_noalloc(C.byref(p), 4, 1, None, fake, fake, fake, hi, fake,
                                       None, None)
    assert st_lo in (1, 5) and st_hi == 8, (lo, hi, st_lo, st_hi)


def test_query_proj_sizes_and_argument_errors(lib):
    wl = WORKLOADS["pro_csa_decode_1m"]
    p = bd.params_for(wl)
    d, d_c = wl.d, wl.d_c
    n1 = -(-(d_c + wl.n_hI) // 128) * 128
    n2 = -(-(wl.n_h * wl.c + wl.n_hI * wl.c_I) // 128) * 128
    assert lib.csa_query_proj_packed_bytes(C.byref(p), d, d_c) == n1 * d * 2 + n2 * d_c * 2
    assert lib.csa_query_proj_workspace_bytes(C.byref(p), 4, d, d_c) == 4 * wl.n_h * wl.c * 4
    assert lib.csa_query_proj_packed_bytes(C.byref(p), d + 32, d_c) == 0  # d % 64
    pf = bd.params_for(WORKLOADS["tiny_csa_prefill_f32"])
    assert lib.csa_query_proj_packed_bytes(C.byref(pf), 512, 128) == 0  # fp32: unsupported
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = 1 << 30
    assert lib.csa_query_proj(C.byref(p), 4, d, d_c, fake, None, fake, fake, fake, fake, fake,
                              fake, ws, None) == 1
    assert lib.csa_query_proj(C.byref(p), 0, d, d_c, fake, fake, fake, fake, fake, fake, fake,
                              fake, ws, None) == 2
    assert lib.csa_query_proj(C.byref(p), 4, d, d_c, fake, fake, fake, fake,
                              C.c_void_p((1 << 20) + 4), fake, fake, fake, ws, None) == 3
    assert lib.csa_query_proj(C.byref(p), 4, d, d_c, fake, fake, fake, fake, fake, fake, fake,
                              fake, 16, None) == 8
    assert lib.csa_query_proj(C.byref(pf), 4, 512, 128, fake, fake, fake, fake, fake, fake,
                              fake, fake, ws, None) == 7


def test_binding_checks_query_proj_tensors(lib):
    import torch
    wl = WORKLOADS["flash_csa_decode_64k"].with_(d=256, d_c=128, n_h=4, c=128, rope_dims=32,
                                                 n_hI=4, c_I=64)
    p = bd.params_for(wl)
    R = 3
    H = torch.zeros(R, 256, dtype=torch.bfloat16)
    pos = torch.zeros(R, dtype=torch.int32)
    packed = torch.zeros(lib.csa_query_proj_packed_bytes(C.byref(p), 256, 128), dtype=torch.uint8)
    cQ = torch.zeros(R, 128, dtype=torch.bfloat16)
    q = torch.zeros(R, 4, 128, dtype=torch.bfloat16)
    qI = torch.zeros(R, 4, 64, dtype=torch.bfloat16)
    w = torch.zeros(R, 4)
    with pytest.raises(ValueError, match=r"^H:"):
        bd.csa_query_proj(p, H.float(), pos, packed, 128, cQ, q, qI, w)
    with pytest.raises(ValueError, match=r"^q:"):
        bd.csa_query_proj(p, H, pos, packed, 128, cQ, q[:2], qI, w)
    with pytest.raises(ValueError, match=r"^w:"):
        bd.csa_query_proj(p, H, pos, packed, 128, cQ, q, qI, w.to(torch.bfloat16))
    with pytest.raises(ValueError, match=r"^packed:"):
        bd.csa_query_proj(p, H, pos, packed[:64], 128, cQ, q, qI, w)
    with pytest.raises(ValueError, match=r"^WUQ:"):
        bd.query_proj_pack(p, torch.zeros(256, 128, dtype=torch.bfloat16),
                           torch.zeros(256, 4, dtype=torch.bfloat16),
                           torch.zeros(128, 100, dtype=torch.bfloat16),
                           torch.zeros(128, 256, dtype=torch.bfloat16))
