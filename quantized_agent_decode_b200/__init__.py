"""Python binding of libqad.so (include/qad.h): argument marshalling only.

Every step of the decode path runs in the CUDA library; this module converts
torch tensors to pointers and return codes to exceptions. There is no CPU
fallback: importing works without a GPU (for the C-ABI export checks), but any
compute call raises if the library or a CUDA device is missing.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqad.so")
_lib = None

QAD_MAX_ROWS = 16
Q4K_BLOCK_BYTES = 144
Q6K_BLOCK_BYTES = 210


class QadError(RuntimeError):
    pass


class ModelDesc(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("hidden", C.c_int), ("inter", C.c_int), ("n_qh", C.c_int),
                ("n_kvh", C.c_int), ("head_dim", C.c_int), ("max_agents", C.c_int), ("kv_cap", C.c_int),
                ("rms_eps", C.c_float), ("w_qkv", C.POINTER(C.c_void_p)), ("w_o", C.POINTER(C.c_void_p)),
                ("w_gu", C.POINTER(C.c_void_p)), ("w_down", C.POINTER(C.c_void_p)),
                ("k_cache", C.POINTER(C.c_void_p)), ("v_cache", C.POINTER(C.c_void_p)), ("kv_format", C.c_int)]


KV_BF16, KV_Q8_0 = 0, 8
SCHED_INTERLEAVE, SCHED_PREFILL_FIRST = 0, 1


class SchedPolicy(C.Structure):
    _fields_ = [("chunk_tokens", C.c_int), ("decode_steps_per_chunk", C.c_int), ("max_decode_rows", C.c_int),
                ("n_draft", C.c_int), ("mode", C.c_int)]


class SchedAgent(C.Structure):
    _fields_ = [("len", C.c_int), ("prompt_left", C.c_int), ("active", C.c_int), ("drafts", C.c_int)]


class AgentRows(C.Structure):
    _fields_ = [("rows", C.c_void_p), ("n_rows", C.c_int), ("len", C.c_int)]


# name -> (restype, argtypes)
SIGNATURES = {
    "qad_last_error": (C.c_char_p, []),
    "qad_version": (C.c_int, []),
    "qad_q4k_unpack": (C.c_int, [C.c_void_p, C.c_longlong] + [C.c_void_p] * 5 + [C.c_void_p]),
    "qad_q6k_unpack": (C.c_int, [C.c_void_p, C.c_longlong] + [C.c_void_p] * 3 + [C.c_void_p]),
    "qad_gemm_ws_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "qad_device_status": (C.c_int, [C.c_int]),
    "qad_debug_stall": (C.c_int, [C.c_int, C.c_int]),
    "qad_q6k_packed_bytes": (C.c_size_t, [C.c_longlong, C.c_int]),
    "qad_q6k_pack": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "qad_q4k_gemm_noalloc_scratch_bytes": (C.c_size_t, []),
    "qad_q4k_gemm_noalloc": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                                       C.c_void_p]),
    "qad_q4k_gemm": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                               C.c_void_p, C.c_size_t, C.c_void_p]),
    "qad_q6k_gemm": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                               C.c_void_p, C.c_size_t, C.c_void_p]),
    "qad_dense_gemm_ws_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "qad_q4k_gemm_dense": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                     C.c_size_t, C.c_void_p]),
    "qad_q6k_gemm_dense": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p,
                                     C.c_size_t, C.c_void_p]),
    "qad_dense_status": (C.c_int, [C.c_int]),
    "qad_prefill_status": (C.c_int, [C.c_int]),
    "qad_verify_ws_bytes": (C.c_size_t, [C.c_int, C.c_int, C.c_int]),
    "qad_verify_step": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_float, C.c_void_p, C.c_int, C.c_void_p, C.c_int]
                        + [C.c_void_p] * 7 + [C.c_size_t, C.c_void_p]),
    "qad_prefill_attn": (C.c_int, [C.c_void_p] * 3 + [C.c_int] * 6 + [C.c_float, C.c_void_p, C.c_void_p]),
    "qad_decode_attn_ws_bytes": (C.c_size_t, [C.c_int] * 5),
    "qad_kv_cache_bytes": (C.c_size_t, [C.c_int] * 5),
    "qad_q8_0_quantize": (C.c_int, [C.c_void_p, C.c_int, C.c_longlong, C.c_void_p, C.c_void_p, C.c_void_p]),
    "qad_decode_attn_q8": (C.c_int, [C.c_void_p] * 7 + [C.c_int] * 6 + [C.c_float, C.c_void_p, C.c_void_p,
                                                                        C.c_size_t, C.c_void_p]),
    "qad_decode_attn": (C.c_int, [C.c_void_p] * 5 + [C.c_int] * 6 + [C.c_float, C.c_void_p, C.c_void_p,
                                                                     C.c_size_t, C.c_void_p]),
    "qad_pack_rows": (C.c_int, [C.POINTER(AgentRows), C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p]),
    "qad_model_create": (C.c_int, [C.POINTER(ModelDesc), C.POINTER(C.c_void_p)]),
    "qad_sched_plan": (C.c_int, [C.POINTER(SchedPolicy), C.POINTER(SchedAgent), C.c_int, C.c_longlong,
                                 C.POINTER(C.c_int), C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    "qad_sched_commit": (C.c_int, [C.POINTER(SchedAgent), C.c_int, C.POINTER(C.c_int), C.c_int, C.c_int,
                                   C.POINTER(C.c_int)]),
    "qad_prompt_lookup": (C.c_int, [C.POINTER(C.c_int), C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_int)]),
    "qad_common_prefix": (C.c_int, [C.POINTER(C.c_int), C.c_int, C.POINTER(C.c_int), C.c_int]),
    "qad_mixed_step_ws_bytes": (C.c_size_t, [C.c_void_p, C.c_int, C.c_int]),
    "qad_mixed_step_debug_bytes": (C.c_size_t, [C.c_void_p, C.c_int, C.c_int]),
    "qad_mixed_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_int,
                                 C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qad_model_destroy": (None, [C.c_void_p]),
    "qad_decode_step_ws_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "qad_decode_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qad_decode_step_host": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int,
                                       C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qad_step_graph_create": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_int,
                                        C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p,
                                        C.POINTER(C.c_void_p)]),
    "qad_step_graph_launch": (C.c_int, [C.c_void_p, C.c_void_p]),
    "qad_step_graph_destroy": (None, [C.c_void_p]),
    "qad_decode_step_launches": (C.c_int, [C.c_void_p]),
    "qad_decode_step_debug_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "qad_model_set_debug": (C.c_int, [C.c_void_p, C.c_void_p, C.c_size_t]),
    "qad_model_set_trace": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int]),
    "qad_model_set_profile": (C.c_int, [C.c_void_p, C.c_int]),
    "qad_model_profile_read": (C.c_int, [C.c_void_p, C.POINTER(C.c_double), C.POINTER(C.c_longlong), C.c_int]),
}

PROFILE_KINDS = ["init", "prep", "gemm_qkv", "attn", "gemm_o", "gemm_gate_up", "gemm_down"]


def lib():
    """Load libqad.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise QadError(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc < 0:
        raise QadError(f"{what} failed ({rc}): {lib().qad_last_error().decode()}")
    return rc


def _dev(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise QadError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise QadError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _require_gpu():
    if not torch.cuda.is_available():
        raise QadError("no CUDA device: the decode path has no CPU fallback")


def alloc_ws(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device workspace (torch allocations are)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def device_status(reset: bool = True) -> int:
    """0 if every GEMM pipeline wait on this device completed since the last reset."""
    return _check(lib().qad_device_status(int(reset)), "qad_device_status")


def debug_stall(kernel: int, at: int) -> None:
    """Test hook: CTA 0 of the skinny GEMM (kernel 0), the dense GEMM (1) or the
    prefill attention (2) stops issuing copies from its step `at` on (at < 0:
    off), so its waits run out."""
    _check(lib().qad_debug_stall(int(kernel), int(at)), "qad_debug_stall")


# ------------------------------------------------------------------ codecs

def q4k_unpack(W: torch.Tensor, n_blocks: int, stream=None):
    _require_gpu()
    dev = W.device
    q = torch.empty(n_blocks, 256, dtype=torch.uint8, device=dev)
    sc = torch.empty(n_blocks, 8, dtype=torch.uint8, device=dev)
    m = torch.empty(n_blocks, 8, dtype=torch.uint8, device=dev)
    d = torch.empty(n_blocks, dtype=torch.int16, device=dev)
    dmin = torch.empty(n_blocks, dtype=torch.int16, device=dev)
    _check(lib().qad_q4k_unpack(_dev(W, "W"), n_blocks, _dev(q, "q"), _dev(sc, "sc"), _dev(m, "m"),
                                _dev(d, "d"), _dev(dmin, "dmin"), _stream(stream)), "qad_q4k_unpack")
    return q, sc, m, d, dmin


def q6k_unpack(W: torch.Tensor, n_blocks: int, stream=None):
    _require_gpu()
    dev = W.device
    q = torch.empty(n_blocks, 256, dtype=torch.uint8, device=dev)
    sc = torch.empty(n_blocks, 16, dtype=torch.int8, device=dev)
    d = torch.empty(n_blocks, dtype=torch.int16, device=dev)
    _check(lib().qad_q6k_unpack(_dev(W, "W"), n_blocks, _dev(q, "q"), _dev(sc, "sc"), _dev(d, "d"),
                                _stream(stream)), "qad_q6k_unpack")
    return q, sc, d


# ------------------------------------------------------------------ GEMM

def gemm_ws_bytes(K: int, M: int) -> int:
    return int(lib().qad_gemm_ws_bytes(K, M))


def _gemm(fn, W, N, K, X, M, Y, accumulate, ws, stream):
    _require_gpu()
    if ws is None:
        ws = alloc_ws(gemm_ws_bytes(K, M), X.device)
    _check(getattr(lib(), fn)(_dev(W, "W"), N, K, _dev(X, "X"), M, _dev(Y, "Y"), int(bool(accumulate)),
                              _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)), fn)
    return Y


def q4k_gemm(W, N, K, X, M, Y, accumulate=False, ws=None, stream=None):
    """Y[M,N] (fp32) = X[M,K] (bf16) @ W^T with W a Q4_K [N, K/256*144] uint8 tensor."""
    return _gemm("qad_q4k_gemm", W, N, K, X, M, Y, accumulate, ws, stream)


def q6k_gemm(W, N, K, X, M, Y, accumulate=False, ws=None, stream=None):
    """Y[M,N] (fp32) = X[M,K] (bf16) @ W^T with W a Q6_K-like matrix in the packed layout (q6k_pack)."""
    return _gemm("qad_q6k_gemm", W, N, K, X, M, Y, accumulate, ws, stream)


def q4k_gemm_noalloc(W, N, K, X, M, Y, accumulate=False, stream=None):
    """q4k_gemm without a workspace: the scratch is the library's fixed device
    array (see qad_q4k_gemm_noalloc in include/qad.h); overlapping calls race."""
    _require_gpu()
    _check(lib().qad_q4k_gemm_noalloc(_dev(W, "W"), N, K, _dev(X, "X"), M, _dev(Y, "Y"), int(bool(accumulate)),
                                      _stream(stream)), "qad_q4k_gemm_noalloc")
    return Y


def dense_gemm_ws_bytes(K: int, M: int) -> int:
    return int(lib().qad_dense_gemm_ws_bytes(K, M))


def prefill_status(reset: bool = True) -> int:
    """0 if every prefill-attention pipeline wait completed since the last reset."""
    return _check(lib().qad_prefill_status(int(reset)), "qad_prefill_status")


def dense_status(reset: bool = True) -> int:
    """0 if every pipeline wait of the dense (prefill) GEMM completed since the last reset."""
    return _check(lib().qad_dense_status(int(reset)), "qad_dense_status")


def _dense(fn, W, N, K, X, M, Y, ws, stream):
    _require_gpu()
    if ws is None:
        ws = alloc_ws(dense_gemm_ws_bytes(K, M), X.device)
    _check(getattr(lib(), fn)(_dev(W, "W"), N, K, _dev(X, "X"), M, _dev(Y, "Y"), _dev(ws, "ws"),
                              ws.numel() * ws.element_size(), _stream(stream)), fn)
    return Y


def q4k_gemm_dense(W, N, K, X, M, Y, ws=None, stream=None):
    """Prefill-chunk GEMM on tcgen05: Y[M,N] (fp32, overwritten) = X[M,K] (bf16) @ W^T, W Q4_K."""
    return _dense("qad_q4k_gemm_dense", W, N, K, X, M, Y, ws, stream)


def q6k_gemm_dense(W, N, K, X, M, Y, ws=None, stream=None):
    """Prefill-chunk GEMM on tcgen05 with W in the packed Q6_K-like layout (q6k_pack)."""
    return _dense("qad_q6k_gemm_dense", W, N, K, X, M, Y, ws, stream)


def q6k_packed_bytes(N: int, K: int) -> int:
    return int(lib().qad_q6k_packed_bytes(N, K))


def q6k_pack(W, N, K, out=None, stream=None):
    """GGUF-layout Q6_K-like blocks (uint8 CUDA tensor [N, K/256*210]) -> packed device layout."""
    _require_gpu()
    if out is None:
        out = torch.empty(q6k_packed_bytes(N, K), dtype=torch.uint8, device=W.device)
    _check(lib().qad_q6k_pack(_dev(W, "W"), N, K, _dev(out, "out"), _stream(stream)), "qad_q6k_pack")
    return out


# ------------------------------------------------------------------ attention

def decode_attn_ws_bytes(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent) -> int:
    return int(lib().qad_decode_attn_ws_bytes(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent))


def decode_attn(Q, Kc, Vc, lens, agent_row_start, n_agents, max_rows_per_agent, kv_cap, n_qh, n_kvh, hd, O,
                scale=None, ws=None, stream=None):
    _require_gpu()
    if scale is None:
        scale = hd ** -0.5
    if ws is None:
        ws = alloc_ws(decode_attn_ws_bytes(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent), Q.device)
    _check(lib().qad_decode_attn(_dev(Q, "Q"), _dev(Kc, "Kc"), _dev(Vc, "Vc"), _dev(lens, "lens"),
                                 _dev(agent_row_start, "agent_row_start"), n_agents, max_rows_per_agent, kv_cap,
                                 n_qh, n_kvh, hd, float(scale), _dev(O, "O"), _dev(ws, "ws"),
                                 ws.numel() * ws.element_size(), _stream(stream)), "qad_decode_attn")
    return O


# ------------------------------------------------------------------ row packer (host)

def verify_ws_bytes(hidden: int, vocab: int, M: int) -> int:
    return int(lib().qad_verify_ws_bytes(hidden, vocab, M))


def verify_step(H, M, hidden, W_head, vocab, agent_row_start, n_agents, row_tokens, lens, out_tokens, n_accept,
                row_argmax=None, logits=None, rms_eps=1e-6, ws=None, stream=None):
    """Logits through the Q4_K head, per-row argmax, greedy draft acceptance and the
    in-place KV-length commit (see qad_verify_step in include/qad.h)."""
    _require_gpu()
    if ws is None:
        ws = alloc_ws(verify_ws_bytes(hidden, vocab, M), H.device)
    opt = lambda t, n: None if t is None else _dev(t, n)  # noqa: E731
    _check(lib().qad_verify_step(_dev(H, "H"), M, hidden, float(rms_eps), _dev(W_head, "W_head"), vocab,
                                 _dev(agent_row_start, "agent_row_start"), n_agents, _dev(row_tokens, "row_tokens"),
                                 _dev(lens, "lens"), _dev(out_tokens, "out_tokens"), _dev(n_accept, "n_accept"),
                                 opt(row_argmax, "row_argmax"), opt(logits, "logits"), _dev(ws, "ws"),
                                 ws.numel() * ws.element_size(), _stream(stream)), "qad_verify_step")
    return out_tokens


def prefill_attn(Q, Kc, Vc, len_, C, kv_cap, n_qh, n_kvh, hd, O, scale=None, stream=None):
    """Causal attention of a C-row prompt chunk at positions len_.. over one agent's cache
    (Kc, Vc bf16 [n_kvh][kv_cap][hd] holding the chunk's k, v); O bf16 [C][n_qh][hd]."""
    _require_gpu()
    if scale is None:
        scale = hd ** -0.5
    _check(lib().qad_prefill_attn(_dev(Q, "Q"), _dev(Kc, "Kc"), _dev(Vc, "Vc"), int(len_), int(C), int(kv_cap),
                                  n_qh, n_kvh, hd, float(scale), _dev(O, "O"), _stream(stream)), "qad_prefill_attn")
    return O


def pack_rows(agent_rows, lens, hidden: int, max_rows: int = QAD_MAX_ROWS):
    """agent_rows: list of CPU bf16 tensors [n_a, hidden] (n_a may be 0).
    Returns (X [M, hidden] bf16, row_agent, row_pos, agent_row_start) as CPU tensors."""
    n = len(agent_rows)
    keep = [r.contiguous() for r in agent_rows]
    arr = (AgentRows * max(n, 1))()
    for a, r in enumerate(keep):
        arr[a].rows = r.data_ptr() if r.numel() else None
        arr[a].n_rows = int(r.shape[0])
        arr[a].len = int(lens[a])
    X = torch.empty(max(max_rows, 1), hidden, dtype=torch.bfloat16)
    ra = torch.empty(max(max_rows, 1), dtype=torch.int32)
    rp = torch.empty(max(max_rows, 1), dtype=torch.int32)
    ars = torch.empty(n + 1, dtype=torch.int32)
    M = _check(lib().qad_pack_rows(arr, n, hidden, max_rows, C.c_void_p(X.data_ptr()),
                                   C.c_void_p(ra.data_ptr()), C.c_void_p(rp.data_ptr()),
                                   C.c_void_p(ars.data_ptr())), "qad_pack_rows")
    return X[:M], ra[:M], rp[:M], ars


def kv_cache_bytes(kv_format, n_agents, n_kvh, kv_cap, hd=128) -> int:
    """Bytes of one K (or V) cache tensor: bf16, or q8_0 codes + (256-aligned) fp16 scales."""
    return int(lib().qad_kv_cache_bytes(kv_format, n_agents, n_kvh, kv_cap, hd))


def q8_cache_planes(buf, n_agents, n_kvh, kv_cap, hd=128):
    """Views (codes int8 [A][n_kvh][cap][hd], scales fp16 bits int16 [A][n_kvh][cap][hd/32]) of a
    uint8 q8_0 cache allocation of kv_cache_bytes(KV_Q8_0, ...) bytes."""
    n = n_agents * n_kvh * kv_cap * hd
    off = (n + 255) // 256 * 256
    codes = buf[:n].view(torch.int8).view(n_agents, n_kvh, kv_cap, hd)
    scales = buf[off:off + n // 16].view(torch.int16).view(n_agents, n_kvh, kv_cap, hd // 32)
    return codes, scales


def q8_0_quantize(x, q=None, d=None, stream=None):
    """q8_0 of a fp32 or bf16 device tensor (numel % 32 == 0): (codes int8, scales fp16 bits int16)."""
    _require_gpu()
    n = x.numel()
    if q is None:
        q = torch.empty(n, dtype=torch.int8, device=x.device)
    if d is None:
        d = torch.empty(n // 32, dtype=torch.int16, device=x.device)
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("q8_0_quantize: x must be float32 or bfloat16")
    _check(lib().qad_q8_0_quantize(_dev(x, "x"), int(x.dtype == torch.bfloat16), n, _dev(q, "q"), _dev(d, "d"),
                                   _stream(stream)), "qad_q8_0_quantize")
    return q, d


def decode_attn_q8(Q, Kq, Kd, Vq, Vd, lens, agent_row_start, n_agents, max_rows_per_agent, kv_cap, n_qh, n_kvh, hd,
                   O, scale=None, ws=None, stream=None):
    _require_gpu()
    if scale is None:
        scale = hd ** -0.5
    if ws is None:
        ws = alloc_ws(decode_attn_ws_bytes(n_agents, n_qh, n_kvh, kv_cap, max_rows_per_agent), Q.device)
    _check(lib().qad_decode_attn_q8(_dev(Q, "Q"), _dev(Kq, "Kq"), _dev(Kd, "Kd"), _dev(Vq, "Vq"), _dev(Vd, "Vd"),
                                    _dev(lens, "lens"), _dev(agent_row_start, "agent_row_start"), n_agents,
                                    max_rows_per_agent, kv_cap, n_qh, n_kvh, hd, float(scale), _dev(O, "O"),
                                    _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
           "qad_decode_attn_q8")
    return O


# ------------------------------------------------------------------ scheduler (host)

def _ints(xs):
    xs = list(xs)
    return (C.c_int * max(len(xs), 1))(*xs)


class Scheduler:
    """Host-side step planner over per-agent states (the C scheduler's state lives here)."""

    def __init__(self, n_agents, chunk_tokens=2048, decode_steps_per_chunk=0, max_decode_rows=12, n_draft=2,
                 mode=SCHED_INTERLEAVE):
        self.policy = SchedPolicy(chunk_tokens, decode_steps_per_chunk, max_decode_rows, n_draft, mode)
        self.agents = (SchedAgent * n_agents)()
        self.n = n_agents
        self.step = 0

    def plan(self):
        """(decode_rows list, chunk_agent or -1, chunk_rows) for the next step."""
        rows = (C.c_int * self.n)()
        ca, cr = C.c_int(), C.c_int()
        _check(lib().qad_sched_plan(C.byref(self.policy), self.agents, self.n, self.step, rows, C.byref(ca),
                                    C.byref(cr)), "qad_sched_plan")
        return list(rows), ca.value, cr.value

    def commit(self, rows, chunk_agent, chunk_rows, n_accept=None):
        acc = _ints(n_accept) if n_accept is not None else None
        _check(lib().qad_sched_commit(self.agents, self.n, _ints(rows), chunk_agent, chunk_rows, acc),
               "qad_sched_commit")
        self.step += 1


def prompt_lookup(tokens, n_draft=2, min_ngram=1, max_ngram=3):
    """Drafts from the latest earlier occurrence of the context's last n-gram (list, possibly empty)."""
    out = (C.c_int * max(n_draft, 1))()
    k = _check(lib().qad_prompt_lookup(_ints(tokens), len(tokens), min_ngram, max_ngram, n_draft, out),
               "qad_prompt_lookup")
    return list(out)[:k]


def common_prefix(a, b) -> int:
    return _check(lib().qad_common_prefix(_ints(a), len(a), _ints(b), len(b)), "qad_common_prefix")


# ------------------------------------------------------------------ model / decode step

class Model:
    """A decoder stack whose weights and KV caches live in caller-owned device tensors."""

    def __init__(self, *, hidden, inter, n_qh, n_kvh, head_dim, max_agents, kv_cap, w_qkv, w_o, w_gu, w_down,
                 k_cache, v_cache, rms_eps=1e-6, kv_format=KV_BF16):
        _require_gpu()
        L = len(w_qkv)
        self._keep = (w_qkv, w_o, w_gu, w_down, k_cache, v_cache)
        arrs = []
        for name, ts in zip(("w_qkv", "w_o", "w_gu", "w_down", "k_cache", "v_cache"), self._keep):
            assert len(ts) == L, name
            arrs.append((C.c_void_p * L)(*[_dev(t, name).value for t in ts]))
        self._arrs = arrs
        d = ModelDesc(L, hidden, inter, n_qh, n_kvh, head_dim, max_agents, kv_cap, rms_eps, *arrs, kv_format)
        h = C.c_void_p()
        _check(lib().qad_model_create(C.byref(d), C.byref(h)), "qad_model_create")
        self.handle = h
        self.n_layers, self.hidden, self.inter = L, hidden, inter
        self.n_qh, self.n_kvh, self.head_dim, self.max_agents, self.kv_cap = n_qh, n_kvh, head_dim, max_agents, kv_cap
        self.kv_format = kv_format
        self._dbg = None

    def close(self):
        if getattr(self, "handle", None):
            lib().qad_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def ws_bytes(self, M: int) -> int:
        return int(lib().qad_decode_step_ws_bytes(self.handle, M))

    def launches(self) -> int:
        return int(lib().qad_decode_step_launches(self.handle))

    def set_debug(self, M: int | None):
        """Attach (M rows) or detach (None) a per-layer intermediates buffer."""
        if M is None:
            self._dbg = None
            _check(lib().qad_model_set_debug(self.handle, None, 0), "qad_model_set_debug")
            return None
        n = int(lib().qad_decode_step_debug_bytes(self.handle, M))
        self._dbg = alloc_ws(n)
        _check(lib().qad_model_set_debug(self.handle, _dev(self._dbg, "dbg"), n), "qad_model_set_debug")
        return self._dbg

    def set_trace(self, enable: bool):
        """Attach (or detach) a per-launch device trace buffer; returns it (int64 [launches][3])."""
        if not enable:
            _check(lib().qad_model_set_trace(self.handle, None, 0), "qad_model_set_trace")
            self._trace = None
            return None
        n = self.launches()
        self._trace = torch.full((n, 3), -1, dtype=torch.int64, device="cuda")
        _check(lib().qad_model_set_trace(self.handle, C.c_void_p(self._trace.data_ptr()), n), "qad_model_set_trace")
        return self._trace

    def trace_reset(self, stream=None):
        self._trace.fill_(-1)

    def trace_read(self):
        """Per launch (start_ns, ready_ns, end_ns) relative to the first start, as a CPU int64 tensor."""
        t = self._trace.cpu()
        end = ~t[:, 2]
        out = torch.stack([t[:, 0], t[:, 1], end], 1)
        return out - out[:, 0].min()

    def set_profile(self, enable: bool):
        _check(lib().qad_model_set_profile(self.handle, int(bool(enable))), "qad_model_set_profile")

    def profile_read(self):
        """{kind: (total_ms, launches)} accumulated since the profiler was enabled."""
        n = len(PROFILE_KINDS)
        ms = (C.c_double * n)()
        cnt = (C.c_longlong * n)()
        _check(lib().qad_model_profile_read(self.handle, ms, cnt, n), "qad_model_profile_read")
        return {k: (ms[i], cnt[i]) for i, k in enumerate(PROFILE_KINDS)}

    def mixed_ws_bytes(self, M: int, C: int) -> int:
        return int(lib().qad_mixed_step_ws_bytes(self.handle, M, C))

    def set_debug_mixed(self, M: int, C: int):
        """Attach a per-layer intermediates buffer sized for a mixed step of M + C rows."""
        n = int(lib().qad_mixed_step_debug_bytes(self.handle, M, C))
        self._dbg = alloc_ws(n)
        _check(lib().qad_model_set_debug(self.handle, _dev(self._dbg, "dbg"), n), "qad_model_set_debug")
        return self._dbg

    def mixed_step(self, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, chunk_agent, chunk_len, C, H_out,
                   ws, stream=None):
        """Decode rows (M) plus a C-row prompt chunk of chunk_agent at positions chunk_len.. (X: decode rows first)."""
        ptr = lambda t, n: _dev(t, n) if t is not None else None  # noqa: E731
        _check(lib().qad_mixed_step(self.handle, _dev(X, "X"), M, ptr(agent_row_start, "agent_row_start"), n_agents,
                                    max_rows_per_agent, ptr(lens, "lens"), chunk_agent, chunk_len, C,
                                    _dev(H_out, "H_out"), _dev(ws, "ws"), ws.numel() * ws.element_size(),
                                    _stream(stream)), "qad_mixed_step")
        return H_out

    def decode_step(self, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws, stream=None):
        _check(lib().qad_decode_step(self.handle, _dev(X, "X"), M, _dev(agent_row_start, "agent_row_start"),
                                     n_agents, max_rows_per_agent, _dev(lens, "lens"), _dev(H_out, "H_out"),
                                     _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
               "qad_decode_step")
        return H_out

    def decode_step_host(self, X_host, M, agent_row_start_host, n_agents, max_rows_per_agent, lens_host, H_host,
                         ws, stream=None):
        """Host tensors in and out (pinned for speed); copies happen inside the call."""
        for t, n in ((X_host, "X"), (agent_row_start_host, "agent_row_start"), (lens_host, "lens"),
                     (H_host, "H_out")):
            if t.is_cuda or not t.is_contiguous():
                raise QadError(f"{n} must be a contiguous host tensor")
        _check(lib().qad_decode_step_host(self.handle, C.c_void_p(X_host.data_ptr()), M,
                                          C.c_void_p(agent_row_start_host.data_ptr()), n_agents,
                                          max_rows_per_agent, C.c_void_p(lens_host.data_ptr()),
                                          C.c_void_p(H_host.data_ptr()), _dev(ws, "ws"),
                                          ws.numel() * ws.element_size(), _stream(stream)), "qad_decode_step_host")
        return H_host

    def graph(self, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws, stream):
        return StepGraph(self, X, M, agent_row_start, n_agents, max_rows_per_agent, lens, H_out, ws, stream)


class StepGraph:
    """A captured decode step (CUDA graph); replay with launch()."""

    def __init__(self, model, X, M, ars, n_agents, max_rows, lens, H_out, ws, stream):
        self.model = model
        self._keep = (X, ars, lens, H_out, ws)
        g = C.c_void_p()
        _check(lib().qad_step_graph_create(model.handle, _dev(X, "X"), M, _dev(ars, "ars"), n_agents, max_rows,
                                           _dev(lens, "lens"), _dev(H_out, "H_out"), _dev(ws, "ws"),
                                           ws.numel() * ws.element_size(), _stream(stream), C.byref(g)),
               "qad_step_graph_create")
        self.handle = g

    def launch(self, stream=None):
        _check(lib().qad_step_graph_launch(self.handle, _stream(stream)), "qad_step_graph_launch")

    def close(self):
        if getattr(self, "handle", None):
            lib().qad_step_graph_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
