"""Thin Python binding of libcsa.so (include/csa.h) through ctypes.

Argument marshalling only: every step of the CSA / HCA forward pass runs in
the library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  There is no fallback: if libcsa.so is missing or fails to load,
every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_F32, CSA_BF16, CSA_KV_FP8MIX = 0, 1, 2
_DT = {"f32": CSA_F32, "bf16": CSA_BF16, "fp8mix": CSA_KV_FP8MIX}
DEV_BAD_INDEX, DEV_BAD_WINDOW, DEV_TIMEOUT, DEV_RANGE = 0x1, 0x2, 0x4, 0x8


class CsaError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class CsaParams(C.Structure):
    _fields_ = [("m", C.c_int), ("overlap", C.c_int), ("c", C.c_int),
                ("rope_dims", C.c_int), ("c_I", C.c_int), ("n_hI", C.c_int),
                ("n_h", C.c_int), ("topk", C.c_int), ("n_win", C.c_int),
                ("rope_base", C.c_float), ("rms_eps", C.c_float),
                ("softmax_scale", C.c_float), ("act", C.c_int), ("kv", C.c_int)]


def params_for(wl) -> CsaParams:
    """csa_params of a configs.Workload."""
    return CsaParams(m=wl.m, overlap=wl.overlap, c=wl.c, rope_dims=wl.rope_dims,
                     c_I=wl.c_I, n_hI=wl.n_hI, n_h=wl.n_h, topk=wl.topk,
                     n_win=wl.n_win, rope_base=wl.rope_base, rms_eps=wl.rms_eps,
                     softmax_scale=wl.softmax_scale, act=_DT[wl.act], kv=_DT[wl.kv])


_lib = None
_vp, _i, _sz = C.c_void_p, C.c_int, C.c_size_t
_P = C.POINTER(CsaParams)

_SIGS = {
    "csa_abi_version": (C.c_int, []),
    "csa_kernel_launches": (C.c_uint64, []),
    "csa_status_string": (C.c_char_p, [C.c_int]),
    "csa_device_status": (C.c_int, [_vp, C.POINTER(C.c_uint32)]),
    "csa_profile_enable": (None, [C.c_int]),
    "csa_profile_kernel_count": (C.c_int, []),
    "csa_profile_kernel_name": (C.c_char_p, [C.c_int]),
    "csa_profile_collect": (C.c_int, [C.POINTER(C.c_double), C.POINTER(C.c_uint64)]),
    "csa_packed_weight_bytes": (_sz, [_P, _i]),
    "csa_pack_weights": (C.c_int, [_P, _i] + [_vp] * 12 + [_vp, _vp]),
    "csa_compress_workspace_bytes": (_sz, [_P, _i, _i, _i]),
    "csa_compress": (C.c_int, [_P, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "hca_compress": (C.c_int, [_P, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "csa_decode_tail_bytes": (_sz, [_P, _i, _i]),
    "csa_decode_append": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp,
                                    _vp, _vp, _i, _vp]),
    "hca_decode_append": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp,
                                    _vp, _i, _vp]),
    "csa_out_proj_packed_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "csa_out_proj_pack": (C.c_int, [_i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "csa_out_proj_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "csa_out_proj": (C.c_int, [_i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "csa_query_proj_packed_bytes": (_sz, [_P, _i, _i]),
    "csa_query_proj_pack": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "csa_query_proj_workspace_bytes": (_sz, [_P, _i, _i, _i]),
    "csa_query_proj": (C.c_int, [_P, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                 _vp]),
    "csa_index_topk_workspace_bytes": (_sz, [_P, _i, _i, _i]),
    "csa_index_topk": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "csa_index_topk_noalloc": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp]),
    "csa_diag_bounded_wait": (C.c_int, [C.c_uint64, _i, _vp, _vp]),
    "csa_mxfp4_quantize": (C.c_int, [_i, _i, _vp, _vp, _vp, _vp]),
    "csa_index_topk_mxfp4": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp,
                                       _sz, _vp]),
    "csa_attend_workspace_bytes": (_sz, [_P, _i, _i, _i]),
    "csa_attend": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _vp, _vp,
                             _vp, _vp, _sz, _vp]),
    "hca_attend": (C.c_int, [_P, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _vp, _vp,
                             _vp, _vp, _sz, _vp]),
}


def lib():
    """The loaded libcsa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library missing: {LIB_PATH} (run "
                               "`python -m long_context_sparse_09_b200.build`)")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return C.c_void_p(t.data_ptr())


def _want(t, dtype, what, min_bytes=0):
    """Argument check of the binding: a tensor of the dtype the call reads,
    holding at least min_bytes (the C ABI sees only the pointer)."""
    if t.dtype != dtype:
        raise ValueError(f"{what}: {dtype} expected, got {t.dtype}")
    if t.numel() * t.element_size() < min_bytes:
        raise ValueError(f"{what}: at least {min_bytes} bytes expected")


def _act(p: CsaParams):
    return torch.float32 if p.act == CSA_F32 else torch.bfloat16


def _esize(p: CsaParams) -> int:
    return 4 if p.act == CSA_F32 else 2


def kv_row_bytes(p: CsaParams) -> int:
    """Bytes of one cache row in the KV format of p."""
    if p.kv == CSA_F32:
        return 4 * p.c
    if p.kv == CSA_BF16:
        return 2 * p.c
    return (p.c - p.rope_dims) + 2 * p.rope_dims


def _want_kv(p: CsaParams, rec, scale, rows: int, what: str):
    """A cache of `rows` rows in the KV format of p (and its scale plane)."""
    if rec is None:
        return
    if p.kv == CSA_KV_FP8MIX:
        _want(rec, torch.uint8, what, rows * kv_row_bytes(p))
        if scale is None:
            raise ValueError(f"{what}_scale: the FP8-mixed format needs its scale plane")
        _want(scale, torch.float32, what + "_scale", rows * 4)
    else:
        _want(rec, torch.float32 if p.kv == CSA_F32 else torch.bfloat16, what,
              rows * kv_row_bytes(p))
        if scale is not None:
            raise ValueError(f"{what}_scale: only the FP8-mixed format has a scale plane")


def _per_seq(n: int, B: int, what: str) -> int:
    if B <= 0 or n % B != 0:
        raise ValueError(f"{what}: {n} rows are not a whole number of rows per sequence "
                         f"for {B} sequences")
    return n // B


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(fn, st):
    if st != 0:
        raise CsaError(fn, st, lib().csa_status_string(st).decode())


def _ws(nbytes, device, workspace):
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def kernel_launches() -> int:
    return int(lib().csa_kernel_launches())


def device_status(stream=None) -> int:
    flags = C.c_uint32(0)
    _check("csa_device_status", lib().csa_device_status(_stream(stream), C.byref(flags)))
    return flags.value


def diag_bounded_wait(limit_ns: int, arrive: bool, waited=None, stream=None):
    """Run the bounded device wait's failure path (arrive False) or its
    completing path (arrive True); waited: optional int64 device tensor of
    one element receiving the ns spent waiting."""
    if waited is not None:
        _want(waited, torch.int64, "waited", 8)
    _check("csa_diag_bounded_wait",
           lib().csa_diag_bounded_wait(int(limit_ns), 1 if arrive else 0, _p(waited),
                                       _stream(stream)))


def profile_enable(on: bool = True):
    lib().csa_profile_enable(1 if on else 0)


def profile_collect() -> dict:
    """{kernel kind: (total device ms, launches)} since the previous collect."""
    n = lib().csa_profile_kernel_count()
    ms = (C.c_double * n)()
    cnt = (C.c_uint64 * n)()
    _check("csa_profile_collect", lib().csa_profile_collect(ms, cnt))
    return {lib().csa_profile_kernel_name(k).decode(): (ms[k], cnt[k]) for k in range(n)}


# ----------------------------------------------------------------- pack --
def csa_pack_weights(p: CsaParams, W: dict, stream=None) -> torch.Tensor:
    """Pack compressor weights ([d][width] each, act dtype) and fp32 biases
    ([m][width]) into the library's layout; returns the packed uint8 buffer."""
    d = W["Wkv_a"].shape[0]
    dev = W["Wkv_a"].device
    nbytes = lib().csa_packed_weight_bytes(C.byref(p), d)
    if nbytes == 0:
        raise CsaError("csa_packed_weight_bytes", 2, "invalid params")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    g = W.get
    st = lib().csa_pack_weights(C.byref(p), d, _p(g("Wkv_a")), _p(g("Wkv_b")), _p(g("Wz_a")),
                                _p(g("Wz_b")), _p(g("WIkv_a")), _p(g("WIkv_b")),
                                _p(g("WIz_a")), _p(g("WIz_b")), _p(g("B_a")), _p(g("B_b")),
                                _p(g("BI_a")), _p(g("BI_b")), _p(packed), _stream(stream))
    _check("csa_pack_weights", st)
    return packed


# ------------------------------------------------------------- compress --
def compress_workspace_bytes(p: CsaParams, B, T, d) -> int:
    return lib().csa_compress_workspace_bytes(C.byref(p), B, T, d)


def _compress_args(p: CsaParams, H, packed, ckv, ckv_scale, kI, win, win_scale):
    """csa_compress / hca_compress read H in the activation dtype and write
    T/m entries (and indexer keys) and T window rows per sequence."""
    B, T, d = H.shape
    _want(H, _act(p), "H")
    _want(packed, torch.uint8, "packed", lib().csa_packed_weight_bytes(C.byref(p), d))
    nE = T // p.m
    _want_kv(p, ckv, ckv_scale, B * nE, "ckv")
    if kI is not None:
        _want(kI, _act(p), "kI", B * nE * p.c_I * _esize(p))
    _want_kv(p, win, win_scale, B * T, "win")


def csa_compress(p: CsaParams, H, packed, ckv, ckv_scale, kI, win, win_scale,
                 workspace=None, stream=None):
    _compress_args(p, H, packed, ckv, ckv_scale, kI, win, win_scale)
    B, T, d = H.shape
    ws, wsb = _ws(compress_workspace_bytes(p, B, T, d), H.device, workspace)
    st = lib().csa_compress(C.byref(p), B, T, d, _p(H), _p(packed), _p(ckv), _p(ckv_scale),
                            _p(kI), _p(win), _p(win_scale), _p(ws), wsb, _stream(stream))
    _check("csa_compress", st)


def hca_compress(p: CsaParams, H, packed, ckv, ckv_scale, win, win_scale,
                 workspace=None, stream=None):
    _compress_args(p, H, packed, ckv, ckv_scale, None, win, win_scale)
    B, T, d = H.shape
    ws, wsb = _ws(compress_workspace_bytes(p, B, T, d), H.device, workspace)
    st = lib().hca_compress(C.byref(p), B, T, d, _p(H), _p(packed), _p(ckv), _p(ckv_scale),
                            _p(win), _p(win_scale), _p(ws), wsb, _stream(stream))
    _check("hca_compress", st)


# ------------------------------------------------------ decode: append --
def decode_tail_bytes(p: CsaParams, B, d) -> int:
    return lib().csa_decode_tail_bytes(C.byref(p), B, d)


def _append_args(p: CsaParams, H, t, tail, win, win_pos0):
    """The decode append reads H in the activation dtype, B int32 positions
    and a tail of decode_tail_bytes; check them (the C ABI sees pointers)."""
    B, d = H.shape
    _want(H, torch.float32 if p.act == CSA_F32 else torch.bfloat16, "H")
    _want(t, torch.int32, "t", B * 4)
    _want(tail, torch.float32, "tail", decode_tail_bytes(p, B, d))
    if win is not None:
        _want(win_pos0, torch.int32, "win_pos0", B * 4)


def csa_decode_append(p: CsaParams, H, t, packed, tail, ckv, ckv_scale, kI, win, win_scale,
                      win_pos0, stream=None):
    """H [B][d] new tokens at positions t [B]; tail from decode_tail_bytes;
    ckv [B][N][row] (ckv_scale [B][N]), kI [B][N][c_I], win [B][W][row]
    (win_scale [B][W]), win_pos0 [B]."""
    _append_args(p, H, t, tail, win, win_pos0)
    B, d = H.shape
    N = ckv.shape[1]
    W = win.shape[1] if win is not None else 0
    st = lib().csa_decode_append(C.byref(p), B, d, _p(H), _p(t), _p(packed), _p(tail), _p(ckv),
                                 _p(ckv_scale), N, _p(kI), _p(win), _p(win_scale), _p(win_pos0),
                                 W, _stream(stream))
    _check("csa_decode_append", st)


def hca_decode_append(p: CsaParams, H, t, packed, tail, ckv, ckv_scale, win, win_scale,
                      win_pos0, stream=None):
    _append_args(p, H, t, tail, win, win_pos0)
    B, d = H.shape
    N = ckv.shape[1]
    W = win.shape[1] if win is not None else 0
    st = lib().hca_decode_append(C.byref(p), B, d, _p(H), _p(t), _p(packed), _p(tail), _p(ckv),
                                 _p(ckv_scale), N, _p(win), _p(win_scale), _p(win_pos0), W,
                                 _stream(stream))
    _check("hca_decode_append", st)


# ------------------------------------------- grouped output projection --
def out_proj_pack(WG, WO, stream=None) -> torch.Tensor:
    """WG [g][c n_h/g][d_g], WO [g d_g][d] (bf16, device) -> the packed
    buffer for csa_out_proj.  n_h and c enter only through c n_h / g, so the
    packing takes n_h = g, c = c n_h / g."""
    g, Kg, d_g = WG.shape
    d = WO.shape[1]
    _want(WG, torch.bfloat16, "WG")
    _want(WO, torch.bfloat16, "WO")
    if WO.shape[0] != g * d_g:
        raise ValueError("WO: [g d_g][d] expected")
    nbytes = lib().csa_out_proj_packed_bytes(g, Kg, g, d_g, d)
    if nbytes == 0:
        raise CsaError("csa_out_proj_packed_bytes", 2, "unsupported shapes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=WG.device)
    st = lib().csa_out_proj_pack(g, Kg, g, d_g, d, _p(WG), _p(WO), _p(packed), _stream(stream))
    _check("csa_out_proj_pack", st)
    return packed


def out_proj_workspace_bytes(R, n_h, c, g, d_g, d) -> int:
    return lib().csa_out_proj_workspace_bytes(R, n_h, c, g, d_g, d)


def csa_out_proj(O, packed, g, d_g, out, workspace=None, stream=None):
    """O [R][n_h][c] bf16 -> out [R][d] bf16 (grouped output projection)."""
    R, n_h, c = O.shape
    d = out.shape[1]
    _want(O, torch.bfloat16, "O")
    _want(out, torch.bfloat16, "out", R * d * 2)
    _want(packed, torch.uint8, "packed", lib().csa_out_proj_packed_bytes(n_h, c, g, d_g, d))
    ws, wsb = _ws(out_proj_workspace_bytes(R, n_h, c, g, d_g, d), O.device, workspace)
    st = lib().csa_out_proj(R, n_h, c, g, d_g, d, _p(O), _p(packed), _p(out), _p(ws), wsb,
                            _stream(stream))
    _check("csa_out_proj", st)


# ------------------------------------------------ query-side projections --
def query_proj_pack(p: CsaParams, WDQ, Ww, WUQ, WIUQ, stream=None) -> torch.Tensor:
    """WDQ [d][d_c], Ww [d][n_hI], WUQ [d_c][n_h c], WIUQ [d_c][n_hI c_I]
    (bf16, device) -> the packed buffer for csa_query_proj."""
    d, d_c = WDQ.shape
    for t, nm, shp in ((WDQ, "WDQ", (d, d_c)), (Ww, "Ww", (d, p.n_hI)),
                       (WUQ, "WUQ", (d_c, p.n_h * p.c)), (WIUQ, "WIUQ", (d_c, p.n_hI * p.c_I))):
        _want(t, torch.bfloat16, nm)
        if tuple(t.shape) != shp:
            raise ValueError(f"{nm}: shape {shp} expected, got {tuple(t.shape)}")
    nbytes = lib().csa_query_proj_packed_bytes(C.byref(p), d, d_c)
    if nbytes == 0:
        raise CsaError("csa_query_proj_packed_bytes", 2, "unsupported shapes")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=WDQ.device)
    st = lib().csa_query_proj_pack(C.byref(p), d, d_c, _p(WDQ), _p(Ww), _p(WUQ), _p(WIUQ),
                                   _p(packed), _stream(stream))
    _check("csa_query_proj_pack", st)
    return packed


def query_proj_workspace_bytes(p: CsaParams, R, d, d_c) -> int:
    return lib().csa_query_proj_workspace_bytes(C.byref(p), R, d, d_c)


def csa_query_proj(p: CsaParams, H, pos, packed, d_c, cQ, q, qI, w, workspace=None,
                   stream=None):
    """H [R][d] bf16 at positions pos [R] -> cQ [R][d_c], q [R][n_h][c],
    qI [R][n_hI][c_I] (bf16) and w [R][n_hI] (fp32)."""
    R, d = H.shape
    _want(H, torch.bfloat16, "H")
    _want(pos, torch.int32, "pos", R * 4)
    _want(packed, torch.uint8, "packed", lib().csa_query_proj_packed_bytes(C.byref(p), d, d_c))
    _want(cQ, torch.bfloat16, "cQ", R * d_c * 2)
    _want(q, torch.bfloat16, "q", R * p.n_h * p.c * 2)
    _want(qI, torch.bfloat16, "qI", R * p.n_hI * p.c_I * 2)
    _want(w, torch.float32, "w", R * p.n_hI * 4)
    ws, wsb = _ws(query_proj_workspace_bytes(p, R, d, d_c), H.device, workspace)
    st = lib().csa_query_proj(C.byref(p), R, d, d_c, _p(H), _p(pos), _p(packed), _p(cQ), _p(q),
                              _p(qI), _p(w), _p(ws), wsb, _stream(stream))
    _check("csa_query_proj", st)


# --------------------------------------------------------- index / top-k --
def index_topk_workspace_bytes(p: CsaParams, B, Q, N) -> int:
    return lib().csa_index_topk_workspace_bytes(C.byref(p), B, Q, N)


def _index_args(p: CsaParams, q_pos, qI, w, kI, idx_out, score_out):
    """Shapes of csa_index_topk's tensors, checked against what the call
    reads and writes; returns (B, Q, N)."""
    B, N = kI.shape[0], kI.shape[1]
    R = qI.shape[0]
    Q = _per_seq(R, B, "qI")
    es = _esize(p)
    _want(qI, _act(p), "qI", R * p.n_hI * p.c_I * es)
    _want(kI, _act(p), "kI", B * N * p.c_I * es)
    _want(w, torch.float32, "w", R * p.n_hI * 4)
    _want(q_pos, torch.int32, "q_pos", R * 4)
    _want(idx_out, torch.int32, "idx_out", R * p.topk * 4)
    if score_out is not None:
        _want(score_out, torch.float32, "score_out", R * p.topk * 4)
    return B, Q, N


def csa_index_topk(p: CsaParams, q_pos, qI, w, kI, idx_out, score_out=None,
                   workspace=None, stream=None):
    """q_pos [B*Q], qI [B*Q][n_hI][c_I], w [B*Q][n_hI], kI [B][N][c_I] ->
    idx_out [B*Q][topk] (and score_out [B*Q][topk])."""
    B, Q, N = _index_args(p, q_pos, qI, w, kI, idx_out, score_out)
    ws, wsb = _ws(index_topk_workspace_bytes(p, B, Q, N), qI.device, workspace)
    st = lib().csa_index_topk(C.byref(p), B, Q, _p(q_pos), _p(qI), _p(w), _p(kI), N,
                              _p(idx_out), _p(score_out), _p(ws), wsb, _stream(stream))
    _check("csa_index_topk", st)


def csa_index_topk_noalloc(p: CsaParams, q_pos, qI, w, kI, idx_out, score_out=None,
                           stream=None):
    """csa_index_topk with the library's fixed scratch instead of a
    workspace (for callers that cannot allocate device memory)."""
    B, Q, N = _index_args(p, q_pos, qI, w, kI, idx_out, score_out)
    st = lib().csa_index_topk_noalloc(C.byref(p), B, Q, _p(q_pos), _p(qI), _p(w), _p(kI), N,
                                      _p(idx_out), _p(score_out), _stream(stream))
    _check("csa_index_topk_noalloc", st)


# -------------------------------------------------------- MXFP4 indexer --
def mxfp4_quantize(x, codes=None, scales=None, stream=None):
    """x [..., width] bf16 (device) -> (codes [..., width/2] uint8, scales
    [..., width/32] uint8) in the MXFP4 format of include/csa.h."""
    _want(x, torch.bfloat16, "x")
    width = x.shape[-1]
    rows = x.numel() // max(width, 1)
    lead = tuple(x.shape[:-1])
    if codes is None:
        codes = torch.empty(lead + (width // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead + (width // 32,), dtype=torch.uint8, device=x.device)
    _want(codes, torch.uint8, "codes", rows * (width // 2))
    _want(scales, torch.uint8, "scales", rows * (width // 32))
    _check("csa_mxfp4_quantize", lib().csa_mxfp4_quantize(rows, width, _p(x), _p(codes),
                                                          _p(scales), _stream(stream)))
    return codes, scales


def csa_index_topk_mxfp4(p: CsaParams, q_pos, qI, w, kI_codes, kI_scales, idx_out,
                         score_out=None, workspace=None, stream=None):
    """csa_index_topk with MXFP4 keys: kI_codes [B][N][c_I/2] and kI_scales
    [B][N][c_I/32] (uint8); q^I is rounded to MXFP4 inside the call and the
    scores are bf16 values."""
    B, N = kI_codes.shape[0], kI_codes.shape[1]
    R = qI.shape[0]
    Q = _per_seq(R, B, "qI")
    _want(qI, torch.bfloat16, "qI", R * p.n_hI * p.c_I * 2)
    _want(w, torch.float32, "w", R * p.n_hI * 4)
    _want(q_pos, torch.int32, "q_pos", R * 4)
    _want(kI_codes, torch.uint8, "kI_codes", B * N * p.c_I // 2)
    _want(kI_scales, torch.uint8, "kI_scales", B * N * p.c_I // 32)
    _want(idx_out, torch.int32, "idx_out", R * p.topk * 4)
    if score_out is not None:
        _want(score_out, torch.float32, "score_out", R * p.topk * 4)
    ws, wsb = _ws(index_topk_workspace_bytes(p, B, Q, N), qI.device, workspace)
    st = lib().csa_index_topk_mxfp4(C.byref(p), B, Q, _p(q_pos), _p(qI), _p(w), _p(kI_codes),
                                    _p(kI_scales), N, _p(idx_out), _p(score_out), _p(ws), wsb,
                                    _stream(stream))
    _check("csa_index_topk_mxfp4", st)


# ---------------------------------------------------------------- attend --
def attend_workspace_bytes(p: CsaParams, B, Q, N) -> int:
    return lib().csa_attend_workspace_bytes(C.byref(p), B, Q, N)


def _attend_args(p: CsaParams, q_pos, q, idx, ckv, ckv_scale, win, win_scale, win_pos0,
                 sink, out):
    """Shapes of csa_attend / hca_attend's tensors, checked against what the
    call reads and writes; returns (B, Q, N, W)."""
    B, N = ckv.shape[0], ckv.shape[1]
    R = q.shape[0]
    Q = _per_seq(R, B, "q")
    W = win.shape[1] if win is not None else 0
    es = _esize(p)
    _want(q, _act(p), "q", R * p.n_h * p.c * es)
    _want(out, _act(p), "out", R * p.n_h * p.c * es)
    _want(q_pos, torch.int32, "q_pos", R * 4)
    _want(sink, torch.float32, "sink", p.n_h * 4)
    if idx is not None:
        _want(idx, torch.int32, "idx", R * p.topk * 4)
    _want_kv(p, ckv, ckv_scale, B * N, "ckv")
    if win is not None:
        if win.shape[0] != B:
            raise ValueError("win: one window per sequence expected")
        _want_kv(p, win, win_scale, B * W, "win")
        _want(win_pos0, torch.int32, "win_pos0", B * 4)
    return B, Q, N, W


def csa_attend(p: CsaParams, q_pos, q, idx, ckv, ckv_scale, win, win_scale, win_pos0,
               sink, out, workspace=None, stream=None):
    """q [B*Q][n_h][c], idx [B*Q][topk], ckv [B][N][row], win [B][W][row] ->
    out [B*Q][n_h][c]."""
    if idx is None:
        raise ValueError("idx: csa_attend attends selected entries")
    B, Q, N, W = _attend_args(p, q_pos, q, idx, ckv, ckv_scale, win, win_scale, win_pos0,
                              sink, out)
    ws, wsb = _ws(attend_workspace_bytes(p, B, Q, N), q.device, workspace)
    st = lib().csa_attend(C.byref(p), B, Q, _p(q_pos), _p(q), _p(idx), _p(ckv), _p(ckv_scale),
                          N, _p(win), _p(win_scale), W, _p(win_pos0), _p(sink), _p(out),
                          _p(ws), wsb, _stream(stream))
    _check("csa_attend", st)


def hca_attend(p: CsaParams, q_pos, q, ckv, ckv_scale, win, win_scale, win_pos0, sink,
               out, workspace=None, stream=None):
    B, Q, N, W = _attend_args(p, q_pos, q, None, ckv, ckv_scale, win, win_scale, win_pos0,
                              sink, out)
    ws, wsb = _ws(attend_workspace_bytes(p, B, Q, N), q.device, workspace)
    st = lib().hca_attend(C.byref(p), B, Q, _p(q_pos), _p(q), _p(ckv), _p(ckv_scale), N,
                          _p(win), _p(win_scale), W, _p(win_pos0), _p(sink), _p(out),
                          _p(ws), wsb, _stream(stream))
    _check("hca_attend", st)
