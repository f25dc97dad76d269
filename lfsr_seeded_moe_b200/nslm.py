"""Thin ctypes binding to libnslm.so, with the names of the C ABI (include/nslm.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  Pointers may be passed as torch tensors (their data_ptr is used) or
as plain integers; a stream may be a torch.cuda.Stream, an integer handle, or
None for torch's current stream.  A negative status raises NslmError.  If
the shared library is missing the import fails loudly: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
# NSLM_LIB_VARIANT loads a variant build of the library from _build/<variant>/:
# l2next or l2basis (`python -m lfsr_seeded_moe_b200.build --stream-source
# l2next`), whose decode kernels read the stream bits from an L2-resident
# 65,536-entry table, or boundscheck (`... build --bounds-check`), whose
# kernels check their indices; NSLM_STREAM_SOURCE is an older name for it.
_SOURCE = os.environ.get("NSLM_LIB_VARIANT", "") or os.environ.get("NSLM_STREAM_SOURCE", "")
LIB_PATH = os.path.join(_HERE, "_build", *([_SOURCE] if _SOURCE else []), "libnslm.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "nslm.h")

NSLM_OK = 0
NSLM_ERR_ARG = -1
NSLM_ERR_ALIGN = -2
NSLM_ERR_SHAPE = -3
NSLM_ERR_WORKSPACE = -4
NSLM_ERR_CUDA = -5
NSLM_ERR_TIMEOUT = -6
NSLM_ERR_UNSUPPORTED = -7

NSLM_P3C5 = 35  # P = 3 with 5-bit coefficients
NSLM_GEMV_FIELDS_READY = 1

NSLM_OP_GEMV = 0
NSLM_OP_GROUPED_GEMM = 1
NSLM_OP_MOE_FFN = 2
NSLM_OP_MOE_STACK = 3
NSLM_OP_MOE_FFN_HYBRID = 4


class NslmError(RuntimeError):
    def __init__(self, name: str, status: int):
        self.status = status
        super().__init__(f"{name} failed: {nslm_status_string(status)} ({status})")


class nslm_seed_matrix(ctypes.Structure):
    _fields_ = [
        ("seeds", ctypes.c_void_p),
        ("coefs", ctypes.c_void_p),
        ("codes", ctypes.c_void_p),
        ("exp_bias", ctypes.c_void_p),
        ("N", ctypes.c_int32),
        ("K", ctypes.c_int32),
        ("P", ctypes.c_int32),
    ]


class nslm_moe_layer(ctypes.Structure):
    _fields_ = [("gate", nslm_seed_matrix), ("up", nslm_seed_matrix), ("down", nslm_seed_matrix)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libnslm.so not found at {LIB_PATH}; build it with `python -m lfsr_seeded_moe_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    mp = ctypes.POINTER(nslm_seed_matrix)
    sig = {
        "nslm_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32, i32]),
        "nslm_seed_gemv": (i32, [mp, vp, i32, vp, vp, sz, vp]),
        "nslm_seed_gemv_flags": (i32, [mp, vp, i32, vp, ctypes.c_uint32, vp]),
        "nslm_seed_grouped_gemm": (i32, [mp, i32, vp, vp, i32, vp, vp, sz, vp]),
        "nslm_moe_route_topk": (i32, [vp, i32, i32, i32, vp, vp, vp]),
        "nslm_moe_seed_ffn": (i32, [mp, mp, mp, i32, vp, vp, vp, i32, i32, vp, vp, sz, vp]),
        "nslm_moe_seed_ffn_hybrid": (i32, [ctypes.POINTER(nslm_moe_layer), i32, ctypes.POINTER(nslm_moe_layer), i32,
                                           vp, vp, vp, i32, i32, vp, vp, sz, vp]),
        "nslm_moe_seed_ffn_static": (i32, [mp, mp, mp, i32, vp, vp, vp, i32, i32, vp, vp]),
        "nslm_moe_stack_decode": (i32, [ctypes.POINTER(nslm_moe_layer), i32, i32, i32, vp, vp, i32,
                                        vp, vp, sz, vp]),
        "nslm_seed_search": (i32, [vp, vp, mp, i32, i32, vp, vp]),
        "nslm_expert_cache_state_bytes": (sz, [i32]),
        "nslm_expert_cache_fetch": (i32, [mp, mp, mp, i32, i32, mp, mp, mp, i32, vp, vp, i32, i32, vp, vp]),
        "nslm_unpack_nibbles": (i32, [vp, mp, vp]),
        "nslm_pack_nibbles": (i32, [mp, vp, vp]),
        "nslm_debug_wait_probe": (i32, [i32, vp, ctypes.c_int64, vp]),
        "nslm_debug_bounds_status": (i32, []),
        "nslm_debug_bounds_probe": (i32, [mp, vp]),
        "nslm_debug_stack_trace": (i32, [vp, sz]),
        "nslm_debug_batched_hidden": (i32, [vp, sz, i32, i32, i32, i32, i32, vp, vp]),
        "nslm_debug_decompress": (i32, [mp, vp, vp]),
        "nslm_debug_decompress_bf16": (i32, [mp, vp, vp]),
        "nslm_device_status": (i32, [vp, vp]),
        "nslm_status_string": (ctypes.c_char_p, [i32]),
        "nslm_last_launch_count": (i32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def declared_functions() -> list[str]:
    """Names of the functions include/nslm.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ \*]*?\b(nslm_[a-z0-9_]+)\s*\(",
                                 text, re.M)))


def _p(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _s(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check(name: str, rc: int) -> int:
    if rc != NSLM_OK:
        raise NslmError(name, rc)
    return rc


def matrix(m) -> nslm_seed_matrix:
    """Marshal an object with seeds/coefs/codes/exp_bias tensors and N, K, P."""
    N = int(m.N) if hasattr(m, "N") else int(m.seeds.shape[0])
    K = int(m.K) if hasattr(m, "K") else int(m.seeds.shape[1]) * 8
    return nslm_seed_matrix(_p(m.seeds), _p(m.coefs), _p(getattr(m, "codes", None)),
                            _p(m.exp_bias), N, K, int(m.P))


def _mat(W):
    return W if isinstance(W, nslm_seed_matrix) else matrix(W)


# ---------------------------------------------------------------- the ABI

def nslm_status_string(status: int) -> str:
    return _lib.nslm_status_string(int(status)).decode()


def nslm_last_launch_count() -> int:
    return int(_lib.nslm_last_launch_count())


def nslm_device_status(ws=None, stream=None) -> int:
    """NSLM_OK or NSLM_ERR_TIMEOUT for the last call that used ws (None: the
    static-scratch entry point).  Waits for the stream; returns the status
    rather than raising on NSLM_ERR_TIMEOUT (other errors raise)."""
    rc = int(_lib.nslm_device_status(_p(ws), _s(stream)))
    if rc not in (NSLM_OK, NSLM_ERR_TIMEOUT):
        raise NslmError("nslm_device_status", rc)
    return rc


def nslm_workspace_bytes(op: int, T: int, E: int, hidden: int, inter: int, k: int, L: int = 0) -> int:
    return int(_lib.nslm_workspace_bytes(op, T, E, hidden, inter, k, L))


def nslm_seed_gemv(W, x_bf16, M: int, y, ws=None, ws_bytes: int = 0, stream=None) -> None:
    _check("nslm_seed_gemv", _lib.nslm_seed_gemv(ctypes.byref(_mat(W)), _p(x_bf16), M, _p(y),
                                                  _p(ws), ws_bytes, _s(stream)))


def nslm_seed_gemv_flags(W, x_bf16, M: int, y, flags: int = 0, stream=None) -> None:
    """nslm_seed_gemv with flags (NSLM_GEMV_FIELDS_READY: W is not written by earlier kernels)."""
    _check("nslm_seed_gemv_flags", _lib.nslm_seed_gemv_flags(ctypes.byref(_mat(W)), _p(x_bf16), M, _p(y),
                                                              int(flags), _s(stream)))


def nslm_seed_grouped_gemm(W, E: int, x_bf16, offsets, R: int, y, ws=None, ws_bytes: int = 0,
                           stream=None) -> None:
    _check("nslm_seed_grouped_gemm",
           _lib.nslm_seed_grouped_gemm(ctypes.byref(_mat(W)), E, _p(x_bf16), _p(offsets), R, _p(y),
                                       _p(ws), ws_bytes, _s(stream)))


def nslm_moe_route_topk(logits, T: int, E: int, k: int, ids, w, stream=None) -> None:
    _check("nslm_moe_route_topk",
           _lib.nslm_moe_route_topk(_p(logits), T, E, k, _p(ids), _p(w), _s(stream)))


def nslm_moe_seed_ffn(gate, up, down, E: int, x_bf16, ids, w, T: int, k: int, y, ws=None,
                      ws_bytes: int = 0, stream=None) -> None:
    _check("nslm_moe_seed_ffn",
           _lib.nslm_moe_seed_ffn(ctypes.byref(_mat(gate)), ctypes.byref(_mat(up)),
                                  ctypes.byref(_mat(down)), E, _p(x_bf16), _p(ids), _p(w), T, k,
                                  _p(y), _p(ws), ws_bytes, _s(stream)))


def nslm_moe_seed_ffn_hybrid(p3, E3: int, p4, E4: int, x_bf16, ids, w, T: int, k: int, y, ws=None,
                             ws_bytes: int = 0, stream=None) -> None:
    """p3 / p4: (gate, up, down) of the P=3 and P=4 expert stacks; ids index E3 + E4 experts."""
    l3 = nslm_moe_layer(*(_mat(m) for m in p3))
    l4 = nslm_moe_layer(*(_mat(m) for m in p4))
    _check("nslm_moe_seed_ffn_hybrid",
           _lib.nslm_moe_seed_ffn_hybrid(ctypes.byref(l3), E3, ctypes.byref(l4), E4, _p(x_bf16), _p(ids), _p(w),
                                         T, k, _p(y), _p(ws), ws_bytes, _s(stream)))


def nslm_moe_seed_ffn_static(gate, up, down, E: int, x_bf16, ids, w, T: int, k: int, y,
                             stream=None) -> None:
    """nslm_moe_seed_ffn without a workspace argument, for callers that may not
    allocate device memory: the library's built-in 1 MiB scratch array is used."""
    _check("nslm_moe_seed_ffn_static",
           _lib.nslm_moe_seed_ffn_static(ctypes.byref(_mat(gate)), ctypes.byref(_mat(up)),
                                         ctypes.byref(_mat(down)), E, _p(x_bf16), _p(ids), _p(w), T,
                                         k, _p(y), _s(stream)))


def moe_layers(layers) -> "ctypes.Array":
    """Marshal a list of (gate, up, down) objects into a host nslm_moe_layer array."""
    arr = (nslm_moe_layer * len(layers))()
    for i, (g, u, d) in enumerate(layers):
        arr[i] = nslm_moe_layer(_mat(g), _mat(u), _mat(d))
    return arr


def nslm_moe_stack_decode(layers, L: int, E: int, k: int, logits, x0_bf16, T: int, y, ws=None,
                          ws_bytes: int = 0, stream=None) -> None:
    arr = layers if isinstance(layers, ctypes.Array) else moe_layers(layers)
    _check("nslm_moe_stack_decode",
           _lib.nslm_moe_stack_decode(arr, L, E, k, _p(logits), _p(x0_bf16), T, _p(y), _p(ws),
                                      ws_bytes, _s(stream)))


def nslm_seed_search(w, out, seed_lo: int = 1, seed_hi: int = 65535, err=None, stream=None, imp=None) -> None:
    """Encode fp32 weights w [N][K] into `out` (seeds/coefs/codes written, exp_bias read);
    imp: optional fp32 [K] importances weighting the error (None: unweighted)."""
    _check("nslm_seed_search", _lib.nslm_seed_search(_p(w), _p(imp), ctypes.byref(_mat(out)), seed_lo,
                                                      seed_hi, _p(err), _s(stream)))


def nslm_expert_cache_state_bytes(slots: int) -> int:
    return int(_lib.nslm_expert_cache_state_bytes(int(slots)))


def nslm_expert_cache_fetch(src, E: int, layer: int, cache, S: int, state, ids, T: int, k: int, slot_ids,
                            stream=None) -> None:
    """src / cache: (gate, up, down) matrices (host-resident source, device slots)."""
    g, u, d = (ctypes.byref(_mat(m)) for m in src)
    gc, uc, dc = (ctypes.byref(_mat(m)) for m in cache)
    _check("nslm_expert_cache_fetch", _lib.nslm_expert_cache_fetch(g, u, d, E, layer, gc, uc, dc, S, _p(state),
                                                                    _p(ids), T, k, _p(slot_ids), _s(stream)))


def nslm_unpack_nibbles(nibbles, out, stream=None) -> None:
    """Write out's coefs (and codes) from a nibbles stream u8 [N][(P+1)*K/16]."""
    _check("nslm_unpack_nibbles", _lib.nslm_unpack_nibbles(_p(nibbles), ctypes.byref(_mat(out)), _s(stream)))


def nslm_pack_nibbles(W, nibbles, stream=None) -> None:
    """Write the nibbles stream u8 [N][(P+1)*K/16] of W's coefs (and codes)."""
    _check("nslm_pack_nibbles", _lib.nslm_pack_nibbles(ctypes.byref(_mat(W)), _p(nibbles), _s(stream)))


def nslm_debug_wait_probe(kind: int, out, cycles: int, stream=None) -> None:
    """Run one bounded device wait (see include/nslm.h) with results in out (5 int32)."""
    _check("nslm_debug_wait_probe", _lib.nslm_debug_wait_probe(int(kind), _p(out), int(cycles), _s(stream)))


def nslm_debug_batched_hidden(ws, ws_bytes: int, T: int, E: int, hidden: int, inter: int, k: int, h_out,
                              stream=None) -> None:
    """bf16 h [T*k][inter] (pair order) left in ws by the last tensor-core FFN call."""
    _check("nslm_debug_batched_hidden",
           _lib.nslm_debug_batched_hidden(_p(ws), ws_bytes, T, E, hidden, inter, k, _p(h_out), _s(stream)))


def nslm_debug_bounds_status() -> int:
    """First bounds-check site recorded since the last call (0: none); bounds-check build only."""
    rc = int(_lib.nslm_debug_bounds_status())
    if rc < 0:
        raise NslmError("nslm_debug_bounds_status", rc)
    return rc


def nslm_debug_stack_trace():
    """The trace build's stamps as a uint64 numpy array [8][256][64] (ns)."""
    import numpy as np
    out = np.zeros((8, 256, 64), np.uint64)
    _check("nslm_debug_stack_trace", _lib.nslm_debug_stack_trace(out.ctypes.data, out.size))
    return out


def nslm_debug_bounds_probe(W, stream=None) -> None:
    _check("nslm_debug_bounds_probe", _lib.nslm_debug_bounds_probe(ctypes.byref(_mat(W)), _s(stream)))


def nslm_debug_decompress(W, w_out, stream=None) -> None:
    _check("nslm_debug_decompress", _lib.nslm_debug_decompress(ctypes.byref(_mat(W)), _p(w_out), _s(stream)))


def nslm_debug_decompress_bf16(W, w_out, stream=None) -> None:
    _check("nslm_debug_decompress_bf16",
           _lib.nslm_debug_decompress_bf16(ctypes.byref(_mat(W)), _p(w_out), _s(stream)))


def raw():
    """The underlying ctypes library (for status-code tests)."""
    return _lib
