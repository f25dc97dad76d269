"""The C ABI on the CPU: the library loads, exports every declared symbol, and
rejects bad arguments with the documented status codes before launching
anything (these checks run on the host; no pointer is dereferenced)."""
import ctypes
import os

import pytest

from lfsr_seeded_moe_b200 import nslm


def test_every_declared_symbol_is_exported():
    names = nslm.declared_functions()
    assert len(names) >= 10
    lib = nslm.raw()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert nslm.nslm_status_string(code) not in ("", "unknown status")
    assert nslm.nslm_status_string(12345) == "unknown status"


def _mat(N=64, K=256, P=4, base=0x10000, codes=True):
    return nslm.nslm_seed_matrix(base, base + 0x100000, base + 0x200000 if codes else 0,
                                 base + 0x300000, N, K, P)


def _gemv(W, x=0x7000000, M=1, y=0x8000000):
    return nslm.raw().nslm_seed_gemv(ctypes.byref(W), x, M, y, 0, 0, 0)


def test_gemv_flags_rejects_unknown_bits():
    rc = nslm.raw().nslm_seed_gemv_flags(ctypes.byref(_mat()), 0x7000000, 1, 0x8000000, 2, 0)
    assert rc == nslm.NSLM_ERR_ARG


def test_gemv_argument_checks():
    assert _gemv(_mat(P=5)) == nslm.NSLM_ERR_SHAPE
    assert _gemv(_mat(K=24, P=4)) == nslm.NSLM_ERR_SHAPE      # P=4 needs K % 16 == 0
    assert _gemv(_mat(K=12, P=3)) == nslm.NSLM_ERR_SHAPE      # K % 8
    assert _gemv(_mat(), M=0) == nslm.NSLM_ERR_SHAPE
    assert _gemv(_mat(), M=9) == nslm.NSLM_ERR_SHAPE
    assert _gemv(_mat(), x=0) == nslm.NSLM_ERR_ARG
    assert _gemv(_mat(), y=0x8000004) == nslm.NSLM_ERR_ALIGN
    assert _gemv(_mat(codes=False)) == nslm.NSLM_ERR_ARG      # P=4 needs codes
    assert _gemv(_mat(base=0x10008)) == nslm.NSLM_ERR_ALIGN
    assert _gemv(_mat(K=65536), M=1) == nslm.NSLM_ERR_SHAPE   # activations exceed shared memory
    assert nslm.raw().nslm_seed_gemv(None, 0x7000000, 1, 0x8000000, 0, 0, 0) == nslm.NSLM_ERR_ARG


def test_ffn_argument_checks():
    E, hidden, inter = 4, 256, 128
    g = _mat(E * inter, hidden)
    u = _mat(E * inter, hidden)
    d = _mat(E * hidden, inter)
    ws_need = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, 1, E, hidden, inter, 2)
    assert ws_need > 0
    f = nslm.raw().nslm_moe_seed_ffn
    ok = dict(x=0x7000000, ids=0x7100000, w=0x7200000, T=1, k=2, y=0x7300000, ws=0x7400000, wsb=ws_need)

    def call(gg=g, uu=u, dd=d, E_=E, **kw):
        a = dict(ok, **kw)
        return f(ctypes.byref(gg), ctypes.byref(uu), ctypes.byref(dd), E_, a["x"], a["ids"], a["w"],
                 a["T"], a["k"], a["y"], a["ws"], a["wsb"], 0)

    assert call(dd=_mat(E * hidden, inter + 8)) == nslm.NSLM_ERR_SHAPE
    assert call(E_=3) == nslm.NSLM_ERR_SHAPE                  # rows not divisible by E
    assert call(k=9) == nslm.NSLM_ERR_SHAPE
    # T > 8 takes the tensor-core path: it needs its own (larger) workspace ...
    assert call(T=9) == nslm.NSLM_ERR_WORKSPACE
    big = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, 9, E, hidden, inter, 2)
    assert big > ws_need
    # ... and hidden / inter multiples of 64
    g72, u72, d72 = _mat(E * 72, hidden), _mat(E * 72, hidden), _mat(E * hidden, 72)
    assert call(gg=g72, uu=u72, dd=d72, T=9, wsb=1 << 30) == nslm.NSLM_ERR_SHAPE
    assert call(wsb=ws_need - 1) == nslm.NSLM_ERR_WORKSPACE
    assert call(ws=0) == nslm.NSLM_ERR_WORKSPACE
    assert call(x=0) == nslm.NSLM_ERR_ARG
    assert call(T=0) == nslm.NSLM_OK                           # nothing to do, nothing launched
    assert nslm.nslm_last_launch_count() == 0


def test_route_argument_checks():
    f = nslm.raw().nslm_moe_route_topk
    assert f(0x1000, 1, 100, 9, 0x2000, 0x3000, 0) == nslm.NSLM_ERR_SHAPE
    assert f(0x1000, 1, 4, 8, 0x2000, 0x3000, 0) == nslm.NSLM_ERR_SHAPE
    assert f(0x1000, 1, 2000, 8, 0x2000, 0x3000, 0) == nslm.NSLM_ERR_SHAPE
    assert f(0, 1, 100, 8, 0x2000, 0x3000, 0) == nslm.NSLM_ERR_ARG


def test_workspace_sizes_are_monotone():
    a = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, 1, 100, 2048, 1408, 8, 45)
    b = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, 8, 100, 2048, 1408, 8, 45)
    assert 0 < a < b
    assert nslm.nslm_workspace_bytes(nslm.NSLM_OP_GEMV, 1, 1, 1, 1, 1) == 0


def test_search_argument_checks():
    f = nslm.raw().nslm_seed_search
    W = _mat(N=4, K=32, P=4)
    w = 0x9000000
    assert f(w, 0, ctypes.byref(W), 0, 10, 0, 0) == nslm.NSLM_ERR_ARG        # seeds start at 1
    assert f(w, 0, ctypes.byref(W), 10, 65536, 0, 0) == nslm.NSLM_ERR_ARG    # 16-bit seeds
    assert f(w, 0, ctypes.byref(W), 20, 10, 0, 0) == nslm.NSLM_ERR_ARG       # empty range
    assert f(0, 0, ctypes.byref(W), 1, 10, 0, 0) == nslm.NSLM_ERR_ARG        # no weights
    assert f(w, 0, ctypes.byref(_mat(N=4, K=24, P=4)), 1, 10, 0, 0) == nslm.NSLM_ERR_SHAPE
    assert f(w, 0, None, 1, 10, 0, 0) == nslm.NSLM_ERR_ARG


def test_nibbles_argument_checks():
    up, pk = nslm.raw().nslm_unpack_nibbles, nslm.raw().nslm_pack_nibbles
    nib = 0x9000000
    assert up(0, ctypes.byref(_mat(N=4, K=32, P=4)), 0) == nslm.NSLM_ERR_ARG
    assert up(nib, None, 0) == nslm.NSLM_ERR_ARG
    assert up(nib, ctypes.byref(_mat(N=4, K=32, P=4, codes=False)), 0) == nslm.NSLM_ERR_ARG
    assert up(nib, ctypes.byref(_mat(N=4, K=24, P=4)), 0) == nslm.NSLM_ERR_SHAPE
    assert pk(ctypes.byref(_mat(N=4, K=32, P=5)), nib, 0) == nslm.NSLM_ERR_SHAPE
    assert pk(ctypes.byref(_mat(N=0, K=32, P=4)), nib, 0) == nslm.NSLM_OK    # empty: nothing to do


def test_expert_cache_argument_checks():
    f = nslm.raw().nslm_expert_cache_fetch
    E, hidden, inter, S = 4, 256, 128, 8
    src = [_mat(E * inter, hidden), _mat(E * inter, hidden), _mat(E * hidden, inter)]
    cac = [_mat(S * inter, hidden, base=0x2000000), _mat(S * inter, hidden, base=0x2000000),
           _mat(S * hidden, inter, base=0x2000000)]
    st, ids, out = 0x9000000, 0x9100000, 0x9200000

    def call(src=src, cac=cac, E_=E, S_=S, T=1, k=4, state=st, layer=0):
        a = [ctypes.byref(m) for m in src]
        c = [ctypes.byref(m) for m in cac]
        return f(*a, E_, layer, *c, S_, state, ids, T, k, out, 0)

    assert nslm.nslm_expert_cache_state_bytes(0) == 0
    assert nslm.nslm_expert_cache_state_bytes(8) > 8 * 8
    assert call(state=0) == nslm.NSLM_ERR_ARG
    assert call(T=3) == nslm.NSLM_ERR_SHAPE                # T * k > S slots
    assert call(S_=4097) == nslm.NSLM_ERR_SHAPE
    assert call(layer=-1) == nslm.NSLM_ERR_SHAPE
    assert call(E_=3) == nslm.NSLM_ERR_SHAPE               # source rows not divisible by E
    assert call(cac=[_mat(S * inter, 512), cac[1], cac[2]]) == nslm.NSLM_ERR_SHAPE   # cache shape differs
    assert call(state=0x9000004) == nslm.NSLM_ERR_ALIGN


def test_p3c5_format_checks():
    # P = 35 (three 5-bit coefficients): K a multiple of 64 and a codes stream;
    # taken by the GEMV, decompression, FFN (decode and tensor-core paths) and
    # grouped GEMM, refused by the search
    assert _gemv(_mat(K=96, P=35)) == nslm.NSLM_ERR_SHAPE
    assert _gemv(_mat(K=128, P=35, codes=False)) == nslm.NSLM_ERR_ARG
    E, hidden, inter = 4, 256, 128
    f = nslm.raw().nslm_moe_seed_ffn
    g, u, d = _mat(E * inter, hidden, P=35), _mat(E * inter, hidden, P=35), _mat(E * hidden, inter, P=35)
    ws = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, 16, E, hidden, inter, 2)
    # both the decode (T <= 8) and the tensor-core (T > 8) paths take the
    # arguments (without a device the call then stops at the device check)
    for T in (1, 16):
        st = f(ctypes.byref(g), ctypes.byref(u), ctypes.byref(d), E, 0x7000000, 0x7100000, 0x7200000, T, 2,
               0x7300000, 0x7400000, ws, 0)
        assert st not in (nslm.NSLM_ERR_SHAPE, nslm.NSLM_ERR_ARG, nslm.NSLM_ERR_ALIGN, nslm.NSLM_ERR_WORKSPACE)
    # a layer mixing formats is refused
    assert f(ctypes.byref(g), ctypes.byref(_mat(E * inter, hidden, P=4)), ctypes.byref(d), E, 0x7000000, 0x7100000,
             0x7200000, 1, 2, 0x7300000, 0x7400000, ws, 0) == nslm.NSLM_ERR_SHAPE
    srch = nslm.raw().nslm_seed_search
    assert srch(0x9000000, 0, ctypes.byref(_mat(N=4, K=64, P=35)), 1, 10, 0, 0) == nslm.NSLM_ERR_SHAPE


def test_wait_probe_argument_checks():
    f = nslm.raw().nslm_debug_wait_probe
    assert f(0, 0, 1000, 0) == nslm.NSLM_ERR_ARG          # no output buffer
    assert f(0, 0x9000000, 0, 0) == nslm.NSLM_ERR_ARG     # no limit
    assert f(4, 0x9000000, 1000, 0) == nslm.NSLM_ERR_ARG  # unknown kind
    assert f(-1, 0x9000000, 1000, 0) == nslm.NSLM_ERR_ARG
    assert f(3, 0x9000004, 1000, 0) == nslm.NSLM_ERR_ALIGN  # the tagged word must be 8-byte aligned


def test_hybrid_argument_checks():
    f = nslm.raw().nslm_moe_seed_ffn_hybrid
    E3, E4, hidden, inter = 3, 4, 256, 128

    def layer(E, P, base):
        return nslm.nslm_moe_layer(_mat(E * inter, hidden, P=P, base=base), _mat(E * inter, hidden, P=P, base=base),
                                   _mat(E * hidden, inter, P=P, base=base))

    l3, l4 = layer(E3, 3, 0x1000000), layer(E4, 4, 0x2000000)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN_HYBRID, 1, E3 + E4, hidden, inter, 2)
    assert wsb > nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, 1, E3 + E4, hidden, inter, 2)

    def call(a=l3, b=l4, e3=E3, e4=E4, ws=0x7400000, n=wsb):
        return f(ctypes.byref(a), e3, ctypes.byref(b), e4, 0x7000000, 0x7100000, 0x7200000, 1, 2, 0x7300000,
                 ws, n, 0)

    assert call(a=l4, b=l3, e3=E4, e4=E3) == nslm.NSLM_ERR_SHAPE   # stacks swapped: P must be 3 then 4
    assert call(e3=0) == nslm.NSLM_ERR_SHAPE
    assert call(n=wsb - 1) == nslm.NSLM_ERR_WORKSPACE
    assert f(None, E3, ctypes.byref(l4), E4, 0x7000000, 0x7100000, 0x7200000, 1, 2, 0x7300000, 0x7400000, wsb,
             0) == nslm.NSLM_ERR_ARG


def test_header_compiles_as_c99(tmp_path):
    # the boundary is a C ABI: its header must be plain C99 (and C++)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "nslm.h"\nint main(void) { nslm_seed_matrix m = {0}; (void)m; return 0; }\n')
    inc = os.path.dirname(nslm.HEADER_PATH)
    for args in (["-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror"], ["-x", "c++", "-std=c++17", "-Wall", "-Werror"]):
        r = subprocess.run([gcc, *args, "-I", inc, "-fsyntax-only", str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr



def test_stack_trace_is_a_trace_build_export():
    # the normal build has no trace: the export refuses without touching its buffer
    import numpy as np
    out = np.zeros(8, np.uint64)
    assert nslm.raw().nslm_debug_stack_trace(out.ctypes.data, out.size) == nslm.NSLM_ERR_UNSUPPORTED
