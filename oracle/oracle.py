"""NumPy driver for the plain-C SeedLM oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA library;
it takes plain NumPy arrays in the documented packed layout:

* ``seeds``    uint16 [N][K/8]  -- one 16-bit LFSR seed per block of 8 weights
* ``coefs``    uint16 [N][K/8]  -- c_j in bits 4j..4j+3 (P=3: code in bits 12..15)
* ``codes``    uint8  [N][K/16] -- P=4 only: block 2m low nibble, 2m+1 high nibble
* ``exp_bias`` int32  [N]       -- per-row exponent bias

(Sources: "K2-Horizon-MoVA-36B-A4B -- NanoSeedLM p4mx-q4v", section "This
upload", for the four tensors; "Qwen3.8-Flash-Next-NanoSeedLM-P4", section
"The family", for 4.5 / 4.0 bits per weight.)  A matrix is any object with
those four attributes plus ``P`` (duck typing, so the oracle imports nothing
from the product).

Functions marked "parity unpinned" have no check against the pages beyond the
readings listed in the C file's header; every other function is pinned by a
CPU test against closed forms, brute force or a library routine.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")


def _u8p_or_null():
    """A pointer type that accepts a uint8 array or None (P=3 has no codes)."""

    class _P:
        @classmethod
        def from_param(cls, obj):
            if obj is None:
                return ctypes.c_void_p(0)
            return _u8p.from_param(obj)

    return _P


_u8n = _u8p_or_null()


def lib():
    """Load (building first if needed) the C oracle."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.nslmo_lfsr_step.restype = ctypes.c_uint16
        L.nslmo_lfsr_step.argtypes = [ctypes.c_uint16]
        L.nslmo_lfsr_period.restype = ctypes.c_int32
        L.nslmo_lfsr_period.argtypes = [ctypes.c_uint16]
        L.nslmo_states.restype = None
        L.nslmo_states.argtypes = [ctypes.c_uint16, ctypes.c_int32, _u16p]
        L.nslmo_basis.restype = None
        L.nslmo_basis.argtypes = [ctypes.c_uint16, ctypes.c_int32, _f64p]
        L.nslmo_regen_block.restype = None
        L.nslmo_regen_block.argtypes = [ctypes.c_uint16, _i32p, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int32, _f64p]
        mat = [_u16p, _u16p, _u8n, _i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.nslmo_decompress_f64.restype = ctypes.c_int32
        L.nslmo_decompress_f64.argtypes = mat + [_f64p]
        L.nslmo_decompress_f32.restype = ctypes.c_int32
        L.nslmo_decompress_f32.argtypes = mat + [_f32p]
        L.nslmo_bf16_to_f64.restype = ctypes.c_double
        L.nslmo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.nslmo_f64_to_bf16.restype = ctypes.c_uint16
        L.nslmo_f64_to_bf16.argtypes = [ctypes.c_double]
        L.nslmo_f64_to_bf16_array.restype = None
        L.nslmo_f64_to_bf16_array.argtypes = [_f64p, ctypes.c_int64, _u16p]
        L.nslmo_seed_matvec.restype = ctypes.c_int32
        L.nslmo_seed_matvec.argtypes = mat + [_u16p, ctypes.c_int32, _f64p]
        L.nslmo_seed_matvec_bf16w.restype = ctypes.c_int32
        L.nslmo_seed_matvec_bf16w.argtypes = mat + [_f64p, ctypes.c_int32, _f64p]
        L.nslmo_route_topk.restype = ctypes.c_int32
        L.nslmo_route_topk.argtypes = [_f32p, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, _i32p, _f64p]
        stk = [_u16p, _u16p, _u8n, _i32p]
        L.nslmo_moe_ffn.restype = ctypes.c_int32
        L.nslmo_moe_ffn.argtypes = stk * 3 + [
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            _u16p, _i32p, _f64p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _f64p]
        L.nslmo_search_block.restype = ctypes.c_int32
        L.nslmo_search_block.argtypes = [
            _f64p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            _i32p, _i32p, _i32p, _f64p]
        L.nslmo_search_block_w.restype = ctypes.c_int32
        L.nslmo_search_block_w.argtypes = [
            _f64p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            _i32p, _i32p, _i32p, _f64p]
        _lib = L
    return _lib


def threads_used() -> int:
    """Threads the OpenMP loops of the oracle run on (OMP_NUM_THREADS or all cores)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


# --------------------------------------------------------------------- LFSR

def lfsr_step(s: int) -> int:
    """One step of the 16-bit Fibonacci LFSR, polynomial x^16+x^14+x^13+x^11+1."""
    return int(lib().nslmo_lfsr_step(s))


def lfsr_period(seed: int) -> int:
    """Steps until the register returns to ``seed`` (65,535 for a maximal LFSR)."""
    return int(lib().nslmo_lfsr_period(seed))


def states(seed: int, n: int) -> np.ndarray:
    """Register states s_0 (= the seed) .. s_{n-1}."""
    out = np.zeros(n, np.uint16)
    lib().nslmo_states(seed, n, out)
    return out


def basis(seed: int, P: int) -> np.ndarray:
    """The 8 x P basis U(seed), U[r][j] = (s_{1+8j+r} - 32768) / 32768."""
    U = np.zeros(8 * P, np.float64)
    lib().nslmo_basis(seed, P, U)
    return U.reshape(8, P)


def regen_block(seed: int, c, code: int, bias: int) -> np.ndarray:
    """w = 2^(code+bias) U(seed) c for one block of 8 weights, exact in fp64."""
    c = np.ascontiguousarray(c, np.int32)
    w = np.zeros(8, np.float64)
    lib().nslmo_regen_block(seed, c, len(c), code, bias, w)
    return w


# ------------------------------------------------------------------ packing

P3C5 = 35  # P = 3 with 5-bit coefficients (see the C oracle for its layout)


def packed_bytes(N: int, K: int, P: int) -> int:
    """Packed bytes of one matrix: streams plus the per-row int32 bias."""
    nb = K // 8
    per_block = {4: 4.5, 3: 4.0, P3C5: 4.375}[P]
    return int(N * nb * per_block) + 4 * N


def _fields(m):
    P = int(m.P)
    seeds = np.ascontiguousarray(m.seeds, np.uint16)
    coefs = np.ascontiguousarray(m.coefs, np.uint16)
    codes = None if P == 3 else np.ascontiguousarray(m.codes, np.uint8)  # P=4: [N][K/16]; P3C5: [N][3K/64]
    eb = np.ascontiguousarray(m.exp_bias, np.int32)
    N = seeds.shape[0]
    K = seeds.shape[1] * 8
    return seeds, coefs, codes, eb, N, K, P


def decompress(m, dtype=np.float32) -> np.ndarray:
    """Dense weights [N][K] of a packed matrix (fp32: exact; fp64 also exact)."""
    seeds, coefs, codes, eb, N, K, P = _fields(m)
    if dtype == np.float64:
        w = np.zeros((N, K), np.float64)
        rc = lib().nslmo_decompress_f64(seeds, coefs, codes, eb, N, K, P, w)
        assert rc == 0, rc
        return w
    w = np.zeros((N, K), np.float32)
    rc = lib().nslmo_decompress_f32(seeds, coefs, codes, eb, N, K, P, w)
    assert rc == 0, "a weight was not exactly representable in fp32"
    return w


# --------------------------------------------------------------------- bf16

def bf16_to_f64(h) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    h = np.asarray(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(v) -> np.ndarray:
    """float64 -> bf16 bit patterns, round to nearest, ties to even."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.zeros(v.shape, np.uint16)
    lib().nslmo_f64_to_bf16_array(v.reshape(-1), v.size, out.reshape(-1))
    return out


def decompress_bf16(m) -> np.ndarray:
    """bf16 bit patterns of the regenerated weights (RNE of the exact value)."""
    return f64_to_bf16(decompress(m, np.float64))


# -------------------------------------------------------------------- matvec

def seed_matvec(m, x_bf16) -> np.ndarray:
    """y[M][N] = x[M][K] W^T in fp64, every weight rebuilt from its seed."""
    seeds, coefs, codes, eb, N, K, P = _fields(m)
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, K)
    M = x.shape[0]
    y = np.zeros((M, N), np.float64)
    rc = lib().nslmo_seed_matvec(seeds, coefs, codes, eb, N, K, P, x, M, y)
    assert rc == 0, rc
    return y


def seed_matvec_bf16w(m, x) -> np.ndarray:
    """As seed_matvec, with each weight rounded to bf16 and x given in fp64."""
    seeds, coefs, codes, eb, N, K, P = _fields(m)
    x = np.ascontiguousarray(x, np.float64).reshape(-1, K)
    M = x.shape[0]
    y = np.zeros((M, N), np.float64)
    rc = lib().nslmo_seed_matvec_bf16w(seeds, coefs, codes, eb, N, K, P, x, M, y)
    assert rc == 0, rc
    return y


def dense_matvec(w, x) -> np.ndarray:
    """The textbook product of a dense matrix and vectors, fp64 (numpy)."""
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64).T


# ------------------------------------------------------------------ routing

def route_topk(logits, k: int):
    """Top-k expert ids (descending logit, ties to the lower id) and the
    softmax of the selected logits, per token."""
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    rc = lib().nslmo_route_topk(logits, T, E, k, ids, w)
    assert rc == 0, rc
    return ids, w


# ---------------------------------------------------------------------- FFN

def silu(g):
    """SiLU(g) = g / (1 + exp(-g)), fp64."""
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def moe_ffn(gate, up, down, E: int, hidden: int, inter: int, x_bf16, ids, w,
            mode: int = 0) -> np.ndarray:
    """Routed expert FFN for T tokens: y_t = sum_q w_tq Down_e(SiLU(Gate_e x) * Up_e x).

    ``gate``/``up``/``down`` are stacks of E experts (rows [e*rows, (e+1)*rows)).
    mode 0 = exact fp64; mode 1 = bf16 weights and bf16 hidden activation
    (the arithmetic of the tensor-core path, mirrored in fp64)."""
    P = int(gate.P)
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, hidden)
    T = x.shape[0]
    ids = np.ascontiguousarray(ids, np.int32).reshape(T, -1)
    k = ids.shape[1]
    w = np.ascontiguousarray(w, np.float64).reshape(T, k)
    y = np.zeros((T, hidden), np.float64)
    args = []
    for m in (gate, up, down):
        s, c, cd, eb, _, _, _ = _fields(m)
        args += [s, c, cd, eb]
    rc = lib().nslmo_moe_ffn(*args, E, hidden, inter, P, x, ids, w, T, k, mode, y)
    assert rc == 0, rc
    return y


def rms_chain(y) -> np.ndarray:
    """The next layer's input in the layer stack: bf16(y / sqrt(mean(y^2) + 1e-6)).

    Reading: the pages run attention between MoE layers, which is out of scope;
    this normalisation keeps the chained activations at unit scale."""
    y = np.asarray(y, np.float64)
    r = np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + 1e-6)
    return f64_to_bf16(y / r)


def layer_stack(layers, logits, x0_bf16, hidden: int, inter: int, E: int, k: int,
                mode: int = 0):
    """Run tokens through a stack of MoE layers.

    ``layers`` is a list of (gate, up, down) stacks, ``logits`` [L][T][E].
    Returns (y of the last layer, list of per-layer inputs as bf16)."""
    x = np.ascontiguousarray(x0_bf16, np.uint16)
    xs = []
    y = None
    for li, (g, u, d) in enumerate(layers):
        xs.append(x)
        ids, w = route_topk(logits[li], k)
        y = moe_ffn(g, u, d, E, hidden, inter, x, ids, w, mode)
        x = rms_chain(y)
    return y, xs


# ------------------------------------------------------------ seed search

def search_block(w8, P: int, bias: int, seed_lo: int = 1, seed_hi: int = 65535, d8=None):
    """Brute-force search of one block: best (seed, c, code, err).

    d8: optional per-weight importances (the mean square of each weight's
    input activation); the error and the least-squares fit are then weighted."""
    w8 = np.ascontiguousarray(w8, np.float64)
    s = np.zeros(1, np.int32)
    c = np.zeros(4, np.int32)
    code = np.zeros(1, np.int32)
    err = np.zeros(1, np.float64)
    if d8 is None:
        rc = lib().nslmo_search_block(w8, P, bias, seed_lo, seed_hi, s, c, code, err)
    else:
        d8 = np.ascontiguousarray(d8, np.float64)
        assert d8.shape == (8,)
        rc = lib().nslmo_search_block_w(w8, d8.ctypes.data, P, bias, seed_lo, seed_hi, s, c, code, err)
    assert rc == 0, rc
    return int(s[0]), c[:P].copy(), int(code[0]), float(err[0])


def normwise_rel_err(y, y_ref) -> float:
    """max_i |y_i - ref_i| / max_i |ref_i| (the 2e-3 gate)."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    den = np.max(np.abs(y_ref))
    if den == 0:
        return float(np.max(np.abs(y)))
    return float(np.max(np.abs(y - y_ref)) / den)


def elementwise_rel_err(y, y_ref, floor: float = 1e-3) -> float:
    """max |dy|/|ref| over entries with |ref| >= floor * max|ref| (reported only)."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    big = np.abs(y_ref) >= floor * np.max(np.abs(y_ref))
    if not np.any(big):
        return 0.0
    return float(np.max(np.abs(y - y_ref)[big] / np.abs(y_ref)[big]))


__all__ = [n for n in dir() if not n.startswith("_")
           and n not in ("np", "math", "ctypes", "os", "annotations")]


# ------------------------------------------------------- the nibbles layout

def blocks_from_streams(m):
    """Per-block fields (c [N][nb][P] signed, code [N][nb]) of a packed matrix in
    this library's streams: c_j in bits 4j..4j+3 of the coefs word; P=4 codes
    in the codes stream (block 2m low nibble, 2m+1 high), P=3 in coefs bits 12..15."""
    seeds, coefs, codes, eb, N, K, P = _fields(m)
    nb = K // 8
    c = np.zeros((N, nb, P), np.int64)
    code = np.zeros((N, nb), np.int64)
    for i in range(N):
        for b in range(nb):
            q = int(coefs[i, b])
            for j in range(P):
                c[i, b, j] = (((q >> (4 * j)) & 0xF) ^ 8) - 8
            if P == 4:
                code[i, b] = (int(codes[i, b // 2]) >> (4 * (b % 2))) & 0xF
            else:
                code[i, b] = (q >> 12) & 0xF
    return c, code


def nibbles_from_blocks(c, code, P: int) -> np.ndarray:
    """The "nibbles" stream of packed rows ([QWEN] "Files": the routed experts are
    NAME.seeds, NAME.nibbles and NAME.exp_bias).  Reading: block b of a row holds
    nibbles (P+1)b .. (P+1)b+P, namely c_0 .. c_{P-1} as two's-complement
    nibbles and then the exponent code; nibble n of a row is in byte n // 2,
    the low half for even n.  That is 2.5 bytes per block for P=4 and 2 for
    P=3, the pages' 4.5 and 4.0 bits per weight with the 16-bit seed."""
    code = np.asarray(code)
    N, nb = code.shape
    out = np.zeros((N, (P + 1) * nb // 2), np.uint8)
    for i in range(N):
        for b in range(nb):
            vals = [int(c[i][b][j]) & 0xF for j in range(P)] + [int(code[i][b])]
            for j, v in enumerate(vals):
                n = (P + 1) * b + j
                out[i, n // 2] |= v << (4 * (n % 2))
    return out


def blocks_from_nibbles(nib, N: int, K: int, P: int):
    """Inverse of nibbles_from_blocks: (c [N][nb][P], code [N][nb])."""
    nib = np.asarray(nib, np.uint8).reshape(N, -1)
    nb = K // 8
    c = np.zeros((N, nb, P), np.int64)
    code = np.zeros((N, nb), np.int64)
    for i in range(N):
        for b in range(nb):
            vals = []
            for j in range(P + 1):
                n = (P + 1) * b + j
                vals.append((int(nib[i, n // 2]) >> (4 * (n % 2))) & 0xF)
            c[i, b] = [(v ^ 8) - 8 for v in vals[:P]]
            code[i, b] = vals[P]
    return c, code
