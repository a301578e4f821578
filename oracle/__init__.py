"""CPU oracle of the CSA / HCA forward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps the plain C reference in
``csa_oracle.c`` (fp64, OpenMP over independent loops) through ctypes and
shares no code with the CUDA library.  Every function takes and returns
numpy float64 arrays holding the exact values of the stored data.

Parity status of each routine (what pins it is listed in the tests):
  compress, norm_rope_rows, index_scores, topk, attend, round_bf16,
  e4m3 encode/decode, fp8mix encode/decode: pinned (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "libcsa_oracle.so")
_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_ip = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_up = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_fp = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "csa_oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = C.CDLL(build())
    lib.ocsa_num_threads.restype = C.c_int
    lib.ocsa_rope.argtypes = [_dp, C.c_int, C.c_double, C.c_double]
    lib.ocsa_rmsnorm.argtypes = [_dp, C.c_int, C.c_double]
    lib.ocsa_matmul.argtypes = [C.c_int, C.c_int, _dp, C.c_int, _dp, _dp]
    lib.ocsa_compress.restype = C.c_int
    lib.ocsa_compress.argtypes = [C.c_int, C.c_int, _dp, C.c_int, C.c_int, C.c_int,
                                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_int, C.c_int,
                                  _dp, C.c_void_p]
    lib.ocsa_norm_rope_rows.argtypes = [C.c_int, C.c_int, C.c_int, C.c_double,
                                        C.c_double, C.c_double, C.c_double, _dp]
    lib.ocsa_nvis.restype = C.c_int
    lib.ocsa_nvis.argtypes = [C.c_int, C.c_int, C.c_int]
    lib.ocsa_index_scores.argtypes = [C.c_int, _ip, C.c_int, C.c_int, _dp, _dp,
                                      C.c_int, _dp, _dp]
    lib.ocsa_topk.argtypes = [C.c_int, C.c_int, _dp, _ip, C.c_int, _ip, _dp]
    lib.ocsa_attend.restype = C.c_int
    lib.ocsa_attend.argtypes = [C.c_int, _ip, C.c_int, C.c_int, C.c_int,
                                C.c_double, C.c_double, _dp, C.c_int, C.c_void_p,
                                C.c_int, C.c_int, _dp, C.c_int, C.c_int, C.c_int,
                                C.c_void_p, _dp, C.c_double, _dp, C.c_void_p]
    lib.ocsa_round_bf16.argtypes = [C.c_int, _dp, _dp]
    lib.ocsa_e2m1_decode.restype = C.c_double
    lib.ocsa_e2m1_decode.argtypes = [C.c_uint8]
    lib.ocsa_mxfp4_encode.argtypes = [C.c_int, _dp, _up, _ip]
    lib.ocsa_mxfp4_decode.argtypes = [C.c_int, _up, _ip, _dp]
    lib.ocsa_group_out_proj.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                        _dp, _dp, _dp, C.c_int, _dp, _dp]
    lib.ocsa_e4m3_decode.restype = C.c_double
    lib.ocsa_e4m3_decode.argtypes = [C.c_uint8]
    lib.ocsa_e4m3_encode.restype = C.c_uint8
    lib.ocsa_e4m3_encode.argtypes = [C.c_float]
    lib.ocsa_fp8mix_encode.argtypes = [C.c_int, C.c_int, C.c_int, _dp, _up, _dp, _fp]
    lib.ocsa_fp8mix_decode.argtypes = [C.c_int, C.c_int, C.c_int, _up, _u16p, _fp, _dp]
    _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a torch tensor (any float dtype)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def num_threads() -> int:
    return _load().ocsa_num_threads()


def rope(x, rope_dims: int, base: float, pos: float) -> np.ndarray:
    """Rotate the last rope_dims of vector x at position pos (negative pos
    de-rotates)."""
    y = _f64(x).copy()
    tail = np.ascontiguousarray(y[len(y) - rope_dims:])
    _load().ocsa_rope(tail, rope_dims, base, pos)
    y[len(y) - rope_dims:] = tail
    return y


def rmsnorm(x, eps: float) -> np.ndarray:
    y = _f64(x).copy()
    _load().ocsa_rmsnorm(y, y.size, eps)
    return y


def matmul(A, W) -> np.ndarray:
    A, W = _f64(A), _f64(W)
    out = np.empty((A.shape[0], W.shape[1]))
    _load().ocsa_matmul(A.shape[0], A.shape[1], A, W.shape[1], W, out)
    return out


def compress(H, m: int, Wkv_a, Wz_a, B_a, Wkv_b=None, Wz_b=None, B_b=None,
             i0: int = 0, i1: int | None = None, want_S: bool = False):
    """Folded entries i0..i1-1 of one sequence H [T][d] (eq. 11-12 when the b
    branch is given, eq. 22-23 otherwise).  Returns out [n][width] (and S
    [n][2m][width] when want_S)."""
    H = _f64(H)
    T, d = H.shape
    overlap = 1 if Wkv_b is not None else 0
    Wkv_a, Wz_a, B_a = _f64(Wkv_a), _f64(Wz_a), _f64(B_a)
    width = Wkv_a.shape[1]
    if overlap:
        Wkv_b, Wz_b, B_b = _f64(Wkv_b), _f64(Wz_b), _f64(B_b)
    if i1 is None:
        i1 = T // m
    n = max(i1 - i0, 0)
    out = np.zeros((n, width))
    S = np.zeros((n, 2 * m, width)) if want_S else None
    rc = _load().ocsa_compress(T, d, H, m, overlap, width, _ptr(Wkv_a), _ptr(Wkv_b),
                               _ptr(Wz_a), _ptr(Wz_b), _ptr(B_a), _ptr(B_b), i0, i1,
                               out, _ptr(S))
    if rc != 0:
        raise ValueError("entry range needs tokens beyond the sequence")
    return (out, S) if want_S else out


def norm_rope_rows(x, rope_dims: int, base: float, eps: float, pos0: float,
                   stride: float) -> np.ndarray:
    """RMSNorm (gain 1) then RoPE of each row; row r at pos0 + stride * r."""
    y = _f64(x).copy()
    n, c = y.shape
    _load().ocsa_norm_rope_rows(n, c, rope_dims, base, eps, pos0, stride, y)
    return y


def nvis(t0: int, m: int, N: int) -> int:
    return _load().ocsa_nvis(int(t0), m, N)


def index_scores(t0s, m: int, qI, w, KI) -> np.ndarray:
    """scores [Q][N] of eq. 16 (-inf where the entry is not visible)."""
    qI, w, KI = _f64(qI), _f64(w), _f64(KI)
    Q, n_hI, c_I = qI.shape
    N = KI.shape[0]
    nv = np.array([nvis(t, m, N) for t in np.asarray(t0s)], dtype=np.int32)
    out = np.empty((Q, N))
    _load().ocsa_index_scores(Q, nv, n_hI, c_I, qI, w, N, KI, out)
    return out


def topk(scores, nv, k: int):
    """(idx [Q][k] ascending, -1 padded; k-th score [Q]) of eq. 17."""
    scores = _f64(scores)
    Q, N = scores.shape
    nv = np.ascontiguousarray(nv, dtype=np.int32)
    idx = np.empty((Q, k), dtype=np.int32)
    kth = np.empty(Q)
    _load().ocsa_topk(Q, N, scores, nv, k, idx, kth)
    return idx, kth


def attend(t0s, q, idx, m: int, kv, n_win: int, win, win_pos0: int, sink,
           rope_dims: int, base: float, scale: float, rope_shift: float = 0.0):
    """out [Q][n_h][c] and total weight mass [Q][n_h] of the shared-KV MQA
    with window and sink; idx None means all visible entries (HCA)."""
    t0s = np.ascontiguousarray(t0s, dtype=np.int32)
    q, kv, sink = _f64(q), _f64(kv), _f64(sink)
    Q, n_h, c = q.shape
    N = kv.shape[0]
    if win is None or n_win == 0:
        win_arr, W = None, 0
    else:
        win_arr = _f64(win)
        W = win_arr.shape[0]
    k = 0
    idx_arr = None
    if idx is not None:
        idx_arr = np.ascontiguousarray(idx, dtype=np.int32)
        k = idx_arr.shape[1]
    out = np.empty((Q, n_h, c))
    mass = np.empty((Q, n_h))
    rc = _load().ocsa_attend(Q, t0s, n_h, c, rope_dims, base, scale, q, k,
                             _ptr(idx_arr), m, N, kv if N else np.zeros((1, c)),
                             n_win, W, int(win_pos0), _ptr(win_arr), sink,
                             rope_shift, out, mass.ctypes.data_as(C.c_void_p))
    if rc != 0:
        raise ValueError("attend: an index or a window row is out of range")
    return out, mass


def group_out_proj(O, WG, WO, round_mid: bool = True):
    """(Y [Q][g d_g], out [Q][d]) of the grouped output projection: O
    [Q][n_h][c], WG [g][c n_h/g][d_g], WO [g d_g][d]."""
    O, WG, WO = _f64(O), _f64(WG), _f64(WO)
    Q, n_h, c = O.shape
    g, Kg, d_g = WG.shape
    d = WO.shape[1]
    if Kg * g != n_h * c or WO.shape[0] != g * d_g or n_h % g:
        raise ValueError("group_out_proj: shapes do not agree")
    Y = np.empty((Q, g * d_g))
    out = np.empty((Q, d))
    _load().ocsa_group_out_proj(Q, n_h, c, g, d_g, d, O, WG, WO, 1 if round_mid else 0, Y, out)
    return Y, out


def e2m1_decode(code: int) -> float:
    return _load().ocsa_e2m1_decode(int(code))


def mxfp4_encode(x):
    """(codes uint8 [n], scale exponents int32 [ceil(n/32)]) of a vector."""
    x = np.ascontiguousarray(_f64(x).reshape(-1))
    codes = np.empty(x.size, dtype=np.uint8)
    exps = np.empty((x.size + 31) // 32, dtype=np.int32)
    _load().ocsa_mxfp4_encode(x.size, x, codes, exps)
    return codes, exps


def mxfp4_decode(codes, exps) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exps = np.ascontiguousarray(exps, dtype=np.int32)
    y = np.empty(codes.size)
    _load().ocsa_mxfp4_decode(codes.size, codes, exps, y)
    return y


def mxfp4_round(x, block_axis_len: int | None = None) -> np.ndarray:
    """The values x takes in MXFP4, blocks of 32 along each row of length
    block_axis_len (default: the last axis)."""
    x = _f64(x)
    n = x.shape[-1] if block_axis_len is None else block_axis_len
    rows = x.reshape(-1, n)
    out = np.empty_like(rows)
    for r in range(rows.shape[0]):
        out[r] = mxfp4_decode(*mxfp4_encode(rows[r]))
    return out.reshape(x.shape)


def round_bf16(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _load().ocsa_round_bf16(x.size, x.reshape(-1), y.reshape(-1))
    return y


def e4m3_decode(code: int) -> float:
    return _load().ocsa_e4m3_decode(int(code))


def e4m3_encode(x: float) -> int:
    return _load().ocsa_e4m3_encode(float(x))


def fp8mix_encode(x, rope_dims: int):
    """(codes [n][c-rope] u8, rope [n][rope] bf16 values as f64, scale [n] f32)."""
    x = _f64(x)
    n, c = x.shape
    codes = np.empty((n, c - rope_dims), dtype=np.uint8)
    rp = np.empty((n, rope_dims))
    sc = np.empty(n, dtype=np.float32)
    _load().ocsa_fp8mix_encode(n, c, rope_dims, x, codes, rp, sc)
    return codes, rp, sc


def fp8mix_decode(codes, rope_bits, scale, c: int, rope_dims: int) -> np.ndarray:
    """Values [n][c] of records given as codes u8, rope bf16 bit patterns u16
    and fp32 scales."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rope_bits = np.ascontiguousarray(rope_bits, dtype=np.uint16)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    n = codes.shape[0]
    x = np.empty((n, c))
    _load().ocsa_fp8mix_decode(n, c, rope_dims, codes, rope_bits, scale, x)
    return x
