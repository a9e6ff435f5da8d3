"""fp64 CPU oracle of the multi-agent decode step (TEST INFRASTRUCTURE ONLY).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg import
this package. The product path (the CUDA library and its binding) never does,
and the two share no code. The arithmetic lives in ``qad_oracle.c``; this file
only builds it, loads it and marshals numpy arrays.

Parity pins for every function are in tests/test_oracle_*.py. The chained
64-layer composition is "parity unpinned" beyond its per-operation pins.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qad_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
i8p = np.ctypeslib.ndpointer(np.int8, flags="C_CONTIGUOUS")
i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile qad_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-Wextra", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        L.orc_half_to_double.restype = C.c_double
        L.orc_half_to_double.argtypes = [C.c_uint16]
        L.orc_bf16_to_double.restype = C.c_double
        L.orc_bf16_to_double.argtypes = [C.c_uint16]
        L.orc_double_to_bf16.restype = C.c_uint16
        L.orc_double_to_bf16.argtypes = [C.c_double]
        L.orc_q4k_decode.argtypes = [u8p, u8p, u8p, u8p, C.POINTER(C.c_uint16), C.POINTER(C.c_uint16)]
        L.orc_q4k_encode.argtypes = [u8p, u8p, u8p, C.c_uint16, C.c_uint16, u8p]
        L.orc_q6k_decode.argtypes = [u8p, u8p, i8p, C.POINTER(C.c_uint16)]
        L.orc_q6k_encode.argtypes = [u8p, i8p, C.c_uint16, u8p]
        L.orc_dequant_matrix.argtypes = [C.c_int, u8p, C.c_int, C.c_int, f64p]
        L.orc_gemm.argtypes = [C.c_int, u8p, C.c_int, C.c_int, u16p, C.c_int, f64p, C.c_void_p, C.c_int]
        L.orc_gemm_rows.argtypes = [C.c_int, u8p, C.c_int, i32p, C.c_int, u16p, C.c_int, f64p, C.c_void_p]
        L.orc_decode_attn.argtypes = [u16p, u16p, u16p, i32p, i32p, C.c_int, C.c_int, C.c_int, C.c_int,
                                      C.c_int, C.c_double, f64p, C.c_void_p, C.c_int]
        L.orc_rmsnorm_bf16.argtypes = [f64p, C.c_int, C.c_int, C.c_double, u16p]
        L.orc_silu_mul_bf16.argtypes = [f64p, f64p, C.c_long, u16p]
        L.orc_pack_rows.restype = C.c_int
        L.orc_pack_rows.argtypes = [C.POINTER(C.c_void_p), i32p, i32p, C.c_int, C.c_int,
                                    u16p, i32p, i32p, i32p]
        L.orc_double_to_half.restype = C.c_uint16
        L.orc_double_to_half.argtypes = [C.c_double]
        L.orc_q8_0_quantize.argtypes = [np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS"), C.c_long, i8p,
                                        u16p]
        L.orc_decode_attn_q8.argtypes = [u16p, i8p, u16p, i8p, u16p, i32p, i32p, C.c_int, C.c_int, C.c_int,
                                         C.c_int, C.c_int, C.c_double, f64p, C.c_void_p, C.c_int]
        L.orc_argmax.restype = C.c_long
        L.orc_argmax.argtypes = [f64p, C.c_long]
        L.orc_accept_greedy.argtypes = [i32p, i32p, i32p, C.c_int, i32p, i32p, i32p]
        L.orc_decode_layer.argtypes = [u8p, u8p, u8p, u8p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                       C.c_double, f64p, C.c_int, i32p, C.c_int, i32p, u16p, u16p,
                                       C.c_int, C.c_int] + [C.c_void_p] * 7
        L.orc_decode_layer_q8.argtypes = [u8p, u8p, u8p, u8p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                          C.c_double, f64p, C.c_int, i32p, C.c_int, i32p, i8p, u16p, i8p, u16p,
                                          C.c_int, C.c_int] + [C.c_void_p] * 7
        L.orc_max_threads.restype = C.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def max_threads() -> int:
    return lib().orc_max_threads()


# ------------------------------------------------------------------ formats

def half_to_double(h: int) -> float:
    return lib().orc_half_to_double(int(h))


def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(int(b))


def double_to_bf16(x: float) -> int:
    return lib().orc_double_to_bf16(float(x))


def bf16_array_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (uint16) to float64 (bit placement only)."""
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_array_to_bf16(a: np.ndarray) -> np.ndarray:
    f = lib().orc_double_to_bf16
    flat = np.asarray(a, np.float64).ravel()
    return np.array([f(float(v)) for v in flat], np.uint16).reshape(np.shape(a))


# ------------------------------------------------------------------ codecs

def q4k_decode(blk: np.ndarray):
    blk = np.ascontiguousarray(blk, np.uint8)
    q, sc, m = np.zeros(256, np.uint8), np.zeros(8, np.uint8), np.zeros(8, np.uint8)
    d, dmin = C.c_uint16(), C.c_uint16()
    lib().orc_q4k_decode(blk, q, sc, m, C.byref(d), C.byref(dmin))
    return q, sc, m, d.value, dmin.value


def q4k_encode(q, sc, m, d: int, dmin: int) -> np.ndarray:
    blk = np.zeros(144, np.uint8)
    lib().orc_q4k_encode(np.ascontiguousarray(q, np.uint8), np.ascontiguousarray(sc, np.uint8),
                         np.ascontiguousarray(m, np.uint8), int(d), int(dmin), blk)
    return blk


def q6k_decode(blk: np.ndarray):
    blk = np.ascontiguousarray(blk, np.uint8)
    q, sc = np.zeros(256, np.uint8), np.zeros(16, np.int8)
    d = C.c_uint16()
    lib().orc_q6k_decode(blk, q, sc, C.byref(d))
    return q, sc, d.value


def q6k_encode(q, sc, d: int) -> np.ndarray:
    blk = np.zeros(210, np.uint8)
    lib().orc_q6k_encode(np.ascontiguousarray(q, np.uint8), np.ascontiguousarray(sc, np.int8), int(d), blk)
    return blk


def dequant(fmt: int, W: np.ndarray, N: int, K: int) -> np.ndarray:
    """fmt 4 = Q4_K, 6 = Q6_K. Returns float64 [N, K]."""
    out = np.zeros((N, K), np.float64)
    lib().orc_dequant_matrix(fmt, np.ascontiguousarray(W, np.uint8).reshape(-1), N, K, out)
    return out


# ------------------------------------------------------------------ GEMM / attention / glue

def gemm(fmt: int, W: np.ndarray, N: int, K: int, X: np.ndarray, nthreads: int = 0):
    """Y, A float64 [M, N]: Y = X W^T, A = |X| |W|^T elementwise-product sums."""
    X = np.ascontiguousarray(X, np.uint16).reshape(-1, K)
    M = X.shape[0]
    Y = np.zeros((M, N), np.float64)
    A = np.zeros((M, N), np.float64)
    lib().orc_gemm(fmt, np.ascontiguousarray(W, np.uint8).reshape(-1), N, K, X, M, Y, _ptr(A),
                   nthreads or max_threads())
    return Y, A


def gemm_rows(fmt: int, W: np.ndarray, K: int, rows, X: np.ndarray):
    """The product for a subset of output rows: Y, A float64 [M, len(rows)]."""
    rows = np.ascontiguousarray(rows, np.int32)
    X = np.ascontiguousarray(X, np.uint16).reshape(-1, K)
    M = X.shape[0]
    Y = np.zeros((M, len(rows)), np.float64)
    A = np.zeros((M, len(rows)), np.float64)
    lib().orc_gemm_rows(fmt, np.ascontiguousarray(W, np.uint8).reshape(-1), K, rows, len(rows), X, M,
                        Y, _ptr(A))
    return Y, A


def decode_attn(Q, Kc, Vc, lens, ars, n_qh, n_kvh, hd, cap, scale=None, nthreads: int = 0):
    """O, B float64 [M, n_qh, hd]."""
    lens = np.ascontiguousarray(lens, np.int32)
    ars = np.ascontiguousarray(ars, np.int32)
    M = int(ars[-1])
    O = np.zeros((M, n_qh, hd), np.float64)
    B = np.zeros((M, n_qh, hd), np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    lib().orc_decode_attn(np.ascontiguousarray(Q, np.uint16).reshape(-1),
                          np.ascontiguousarray(Kc, np.uint16).reshape(-1),
                          np.ascontiguousarray(Vc, np.uint16).reshape(-1),
                          lens, ars, len(lens), cap, n_qh, n_kvh, hd, float(scale), O, _ptr(B),
                          nthreads or max_threads())
    return O, B


def rmsnorm_bf16(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    h = np.ascontiguousarray(h, np.float64)
    M, H = h.shape
    out = np.zeros((M, H), np.uint16)
    lib().orc_rmsnorm_bf16(h, M, H, eps, out)
    return out


def silu_mul_bf16(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(g, np.float64)
    u = np.ascontiguousarray(u, np.float64)
    out = np.zeros(g.shape, np.uint16)
    lib().orc_silu_mul_bf16(g.reshape(-1), u.reshape(-1), g.size, out.reshape(-1))
    return out


def pack_rows(agent_rows, lens, H: int):
    """agent_rows: list of uint16 [n_a, H] arrays (n_a may be 0)."""
    n = len(agent_rows)
    arrs = [np.ascontiguousarray(a, np.uint16).reshape(-1, H) for a in agent_rows]
    ptrs = (C.c_void_p * max(n, 1))(*[a.ctypes.data for a in arrs])
    n_rows = np.array([a.shape[0] for a in arrs], np.int32)
    M = int(n_rows.sum())
    X = np.zeros((max(M, 1), H), np.uint16)
    ra, rp = np.zeros(max(M, 1), np.int32), np.zeros(max(M, 1), np.int32)
    ars = np.zeros(n + 1, np.int32)
    m = lib().orc_pack_rows(ptrs, n_rows, np.ascontiguousarray(lens, np.int32), n, H, X, ra, rp, ars)
    assert m == M
    return X[:M], ra[:M], rp[:M], ars


def double_to_half(x: float) -> int:
    return int(lib().orc_double_to_half(float(x)))


def q8_0_quantize(x: np.ndarray):
    """float32 [..., n] (n % 32 == 0) -> (int8 codes [..., n], fp16 scale bits [..., n / 32])."""
    x = np.ascontiguousarray(x, np.float32)
    q = np.zeros(x.shape, np.int8)
    d = np.zeros(x.shape[:-1] + (x.shape[-1] // 32,), np.uint16)
    lib().orc_q8_0_quantize(x.reshape(-1), x.size, q.reshape(-1), d.reshape(-1))
    return q, d


def decode_attn_q8(Q, Kq, Kd, Vq, Vd, lens, ars, n_qh, n_kvh, hd, cap, scale=None, nthreads: int = 0):
    """Attention over a q8_0 cache: O, B float64 [M, n_qh, hd]."""
    lens = np.ascontiguousarray(lens, np.int32)
    ars = np.ascontiguousarray(ars, np.int32)
    M = int(ars[-1])
    O = np.zeros((M, n_qh, hd), np.float64)
    B = np.zeros((M, n_qh, hd), np.float64)
    lib().orc_decode_attn_q8(np.ascontiguousarray(Q, np.uint16).reshape(-1),
                             np.ascontiguousarray(Kq, np.int8).reshape(-1), np.ascontiguousarray(Kd, np.uint16).reshape(-1),
                             np.ascontiguousarray(Vq, np.int8).reshape(-1), np.ascontiguousarray(Vd, np.uint16).reshape(-1),
                             lens, ars, len(lens), cap, n_qh, n_kvh, hd, 1.0 / np.sqrt(hd) if scale is None else float(scale),
                             O.reshape(-1), _ptr(B.reshape(-1)), nthreads or max_threads())
    return O, B


def argmax(v: np.ndarray) -> int:
    """First index of the maximum of a 1-D float64 array."""
    v = np.ascontiguousarray(v, np.float64)
    return int(lib().orc_argmax(v, v.size))


def accept_greedy(row_argmax, row_tokens, ars, lens):
    """Greedy draft acceptance: returns (new lens, out_tokens, n_accept)."""
    ars = np.ascontiguousarray(ars, np.int32)
    n = len(ars) - 1
    M = int(ars[-1])
    lens2 = np.array(lens, np.int32, copy=True)
    out = np.zeros(max(M, 1), np.int32)
    acc = np.zeros(max(n, 1), np.int32)
    lib().orc_accept_greedy(np.ascontiguousarray(row_argmax, np.int32).reshape(-1) if M else np.zeros(1, np.int32),
                            np.ascontiguousarray(row_tokens, np.int32).reshape(-1) if M else np.zeros(1, np.int32),
                            ars, n, lens2, out, acc)
    return lens2, out[:M], acc[:n]


def decode_layer(Wqkv, Wo, Wgu, Wdown, H, I, n_qh, n_kvh, hd, h, ars, lens, Kc, Vc, cap,
                 eps=1e-6, nthreads: int = 0, want=False):
    """One layer on the fp64 residual ``h`` [M, H] (in place); caches updated in place.
    Kc, Vc are bf16 arrays, or (codes int8, scales fp16 bits) pairs for a q8_0 cache.
    With want=True also returns the intermediates dict."""
    M = h.shape[0]
    nq, nkv = n_qh * hd, n_kvh * hd
    inter = {}
    if want:
        inter = dict(x1=np.zeros((M, H), np.uint16), qkv=np.zeros((M, nq + 2 * nkv), np.float64),
                     attn=np.zeros((M, nq), np.uint16), hmid=np.zeros((M, H), np.float64),
                     x2=np.zeros((M, H), np.uint16), gu=np.zeros((M, 2 * I), np.float64),
                     act=np.zeros((M, I), np.uint16))
    names = ["x1", "qkv", "attn", "hmid", "x2", "gu", "act"]
    ptrs = [_ptr(inter.get(k)) for k in names]
    W = [np.ascontiguousarray(w, np.uint8).reshape(-1) for w in (Wqkv, Wo, Wgu, Wdown)]
    common = (H, I, n_qh, n_kvh, hd, eps, h, M, np.ascontiguousarray(ars, np.int32), len(lens),
              np.ascontiguousarray(lens, np.int32))
    if isinstance(Kc, tuple):
        for a in (*Kc, *Vc):
            assert a.flags["C_CONTIGUOUS"]  # updated in place
        lib().orc_decode_layer_q8(*W, *common, Kc[0].reshape(-1), Kc[1].reshape(-1), Vc[0].reshape(-1),
                                  Vc[1].reshape(-1), cap, nthreads or max_threads(), *ptrs)
    else:
        lib().orc_decode_layer(*W, *common, Kc.reshape(-1), Vc.reshape(-1), cap, nthreads or max_threads(),
                               *ptrs)
    return inter


def prompt_lookup(tokens, min_ngram, max_ngram, n_draft):
    """Prompt-lookup drafts, written out: for n from max_ngram down to min_ngram,
    every earlier position j whose n tokens equal the context's last n tokens
    and that is followed by at least one token is a match; the latest match
    wins and its following tokens (up to n_draft) are the drafts."""
    T = list(tokens)
    for n in range(max_ngram, min_ngram - 1, -1):
        if n >= len(T):
            continue
        suffix = T[len(T) - n:]
        matches = [j for j in range(0, len(T) - n) if T[j:j + n] == suffix]
        if matches:
            j = max(matches)
            return T[j + n:j + n + n_draft]
    return []
