"""CPU tests of the C ABI: the library loads, exports every symbol that
include/wall.h declares, and rejects bad arguments on the host before any
launch (no GPU needed for any of these calls)."""
import ctypes
import os
import re

import pytest

from channel_decay_softmax_b200 import _lib as L
from channel_decay_softmax_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wall.h")

FAKE = 4096  # an aligned, never dereferenced address: every call below fails its checks first


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(wall_\w+)\s*\(", src,
                                 flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from channel_decay_softmax_b200 import build
    build.build()
    return L.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTS)


def test_version_and_error_strings(lib):
    assert lib.wall_version() >= 1
    for code, word in ((0, b"ok"), (1, b"invalid"), (2, b"unsupported"), (3, b"CUDA"),
                       (4, b"timed out")):
        assert word in lib.wall_error_string(code)


def _fwd(lib, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, P=FAKE, dtype=0, B=1, T=16, H=2, HQ=4, K=64, V=64,
             scale=0.0, gs=None, sink=None, window=0, cu=None, n_seq=0, o=FAKE, lse=FAKE,
             ws=None, ws_bytes=0, stream=None)
    a.update(over)
    return lib.wall_attn_fwd(a["q"], a["k"], a["v"], a["P"], a["dtype"], a["B"], a["T"], a["H"],
                             a["HQ"], a["K"], a["V"], a["scale"], a["gs"], a["sink"],
                             a["window"], a["cu"], a["n_seq"], a["o"], a["lse"], a["ws"],
                             a["ws_bytes"], a["stream"])


def test_fwd_rejects_bad_arguments(lib):
    assert _fwd(lib, HQ=3) == L.WALL_ERR_INVALID_ARG            # HQ % H != 0
    assert _fwd(lib, H=0) == L.WALL_ERR_INVALID_ARG
    assert _fwd(lib, dtype=5) == L.WALL_ERR_INVALID_ARG
    assert _fwd(lib, K=100) == L.WALL_ERR_UNSUPPORTED           # not a multiple of 8
    assert _fwd(lib, V=256) == L.WALL_ERR_UNSUPPORTED
    assert _fwd(lib, q=None) == L.WALL_ERR_INVALID_ARG
    assert _fwd(lib, q=FAKE + 4) == L.WALL_ERR_INVALID_ARG      # misaligned
    assert _fwd(lib, B=2, cu=FAKE, n_seq=1) == L.WALL_ERR_INVALID_ARG  # varlen needs B == 1
    # g_scalar needs workspace; none given
    assert _fwd(lib, gs=FAKE) == L.WALL_ERR_INVALID_ARG
    assert _fwd(lib, T=0) == L.WALL_OK                          # empty: nothing to do


def test_bwd_rejects_bad_arguments(lib):
    def bwd(**over):
        a = dict(dO=FAKE, gs=None, dgs=None, sink=None, dsink=None, ws=None, ws_bytes=0, T=16,
                 HQ=4, fws=None)
        a.update(over)
        return lib.wall_attn_bwd(a["dO"], FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, a["T"], 2,
                                 a["HQ"], 64, 64, 0.0, a["gs"], a["sink"], 0, None, 0, FAKE,
                                 FAKE, FAKE, FAKE, a["dgs"], a["dsink"], a["ws"], a["ws_bytes"],
                                 a["fws"], None)
    assert bwd(HQ=5) == L.WALL_ERR_INVALID_ARG
    assert bwd(gs=FAKE) == L.WALL_ERR_INVALID_ARG               # dg_scalar missing
    assert bwd(dgs=FAKE) == L.WALL_ERR_INVALID_ARG              # g_scalar missing
    assert bwd(dO=None) == L.WALL_ERR_INVALID_ARG
    assert bwd() == L.WALL_ERR_INVALID_ARG                      # no workspace
    assert bwd(ws=FAKE, ws_bytes=16) == L.WALL_ERR_INVALID_ARG  # workspace too small
    assert bwd(fws=FAKE + 4) == L.WALL_ERR_INVALID_ARG          # misaligned forward workspace


def test_cache_and_decode_reject_bad_arguments(lib):
    kc = lib.wall_build_kv_cache
    assert kc(FAKE, FAKE, 0, 1, 10, 2, 4, 64, 64, 0, FAKE, FAKE, 9, None) == L.WALL_ERR_INVALID_ARG
    assert kc(FAKE, FAKE, 0, 1, 10, 2, 4, 64, 0, 0, FAKE, FAKE, 10, None) == L.WALL_ERR_INVALID_ARG
    assert kc(FAKE, FAKE, 0, 1, 10, 2, 4, 60, 64, 0, FAKE, FAKE, 10, None) == L.WALL_ERR_UNSUPPORTED
    assert kc(FAKE, FAKE, 0, 1, 0, 2, 4, 64, 64, 0, FAKE, FAKE, 10, None) == L.WALL_OK
    dec = lib.wall_attn_decode
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.0, 64, 0, 1]
    # T_kv = 0 is invalid: the current token's key must be cached
    assert dec(*args, 0, 10, 2, 4, 64, 64, FAKE, FAKE, FAKE, 1 << 20, None) == L.WALL_ERR_INVALID_ARG
    # T_kv beyond capacity
    assert dec(*args, 11, 10, 2, 4, 64, 64, FAKE, FAKE, FAKE, 1 << 20, None) == L.WALL_ERR_INVALID_ARG
    # group of 64 query heads per kv head is beyond the decode kernel
    assert dec(*args, 10, 10, 1, 64, 64, 64, FAKE, FAKE, FAKE, 1 << 20, None) == L.WALL_ERR_UNSUPPORTED
    # workspace too small
    assert dec(*args, 10, 10, 2, 4, 64, 64, FAKE, FAKE, FAKE, 8, None) == L.WALL_ERR_INVALID_ARG


def test_decode_step_rejects_bad_arguments(lib):
    st = lib.wall_decode_step
    B, Tcap, H, HQ, K, V, C = 2, 256, 2, 8, 128, 128, 64
    need = lib.wall_decode_step_workspace(B, Tcap, H, HQ, V, C)
    # the counters follow the split partials sized for the capacity
    al = lambda x: (x + 255) // 256 * 256
    assert need > al(4 * B * HQ) and (need - al(4 * B * HQ)) % 256 == 0

    def call(dtype=0, t=10, C=C, H=H, HQ=HQ, K=K, V=V, ws_bytes=need, q=FAKE, kt=FAKE,
             carry=FAKE):
        return st(q, FAKE, FAKE, FAKE, dtype, carry, kt, FAKE, FAKE, None, 0.0, C, t, B, Tcap,
                  H, HQ, K, V, FAKE, None, FAKE, ws_bytes, None)

    assert call(dtype=2) == L.WALL_ERR_INVALID_ARG           # unknown dtype
    assert call(t=-1) == L.WALL_ERR_INVALID_ARG              # before the sequence
    assert call(t=Tcap) == L.WALL_ERR_INVALID_ARG            # no room to append
    assert call(dtype=1) == L.WALL_ERR_UNSUPPORTED           # fp32: three-call path instead
    assert call(K=96) == L.WALL_ERR_UNSUPPORTED              # head size outside {64, 128}
    assert call(C=48) == L.WALL_ERR_UNSUPPORTED              # chunk not a multiple of 32
    assert call(H=1, HQ=16) == L.WALL_ERR_UNSUPPORTED        # 16 query heads per kv head
    assert call(q=None) == L.WALL_ERR_INVALID_ARG
    assert call(kt=FAKE + 8) == L.WALL_ERR_INVALID_ARG       # misaligned cache
    assert call(carry=None) == L.WALL_ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == L.WALL_ERR_INVALID_ARG  # workspace too small
    assert lib.wall_decode_step_workspace(1, 0, 1, 1, 64, 64) == 0


def test_decode_chunk_rejects_bad_arguments(lib):
    ch = lib.wall_attn_decode_chunk
    wsf = lib.wall_attn_decode_chunk_workspace
    B, Tq, T_kv, Tcap, H, HQ, K, V, C = 2, 64, 1000, 1024, 2, 8, 128, 128, 64
    al = lambda x: (x + 255) // 256 * 256
    # tensor-core path: anchored queries (bf16) and 128-row block anchors (fp32)
    tc = al(2 * B * Tq * HQ * K) + al(4 * B * 1 * HQ * K)
    assert wsf(0, B, Tq, T_kv, H, HQ, K, V, C) == tc
    # split path (fp32): per query row and split, the partial (o, m, l)
    split = wsf(1, B, Tq, T_kv, H, HQ, K, V, C)
    assert split > 0 and split % (4 * B * Tq * HQ * (V + 2)) < 256
    assert wsf(0, B, Tq + 1, Tq, H, HQ, K, V, C) == 0          # more queries than positions

    def call(dtype=0, Tq=Tq, T_kv=T_kv, Tcap=Tcap, C=C, H=H, HQ=HQ, K=K, V=V, ws_bytes=tc,
             q=FAKE, kt=FAKE, B=B):
        return ch(q, FAKE, FAKE, kt, FAKE, None, 0.0, C, dtype, B, Tq, T_kv, Tcap, H, HQ, K, V,
                  FAKE, None, FAKE, ws_bytes, None)

    assert call(dtype=3) == L.WALL_ERR_INVALID_ARG
    assert call(Tq=T_kv + 1) == L.WALL_ERR_INVALID_ARG        # queries past the cache
    assert call(Tcap=T_kv - 1) == L.WALL_ERR_INVALID_ARG      # cache shorter than T_kv
    assert call(T_kv=0, Tq=0) == L.WALL_ERR_INVALID_ARG
    assert call(HQ=7) == L.WALL_ERR_INVALID_ARG               # HQ % H != 0
    assert call(K=136) == L.WALL_ERR_UNSUPPORTED              # head size beyond 128
    assert call(H=1, HQ=64) == L.WALL_ERR_UNSUPPORTED         # 64 query heads per kv head
    assert call(q=None) == L.WALL_ERR_INVALID_ARG
    assert call(kt=FAKE + 4) == L.WALL_ERR_INVALID_ARG        # misaligned cache
    assert call(ws_bytes=tc - 1) == L.WALL_ERR_INVALID_ARG    # workspace too small
    assert call(dtype=1, ws_bytes=tc) == L.WALL_ERR_INVALID_ARG  # fp32 needs the split partials
    assert call(dtype=1, Tq=700, T_kv=700, B=100) == L.WALL_ERR_UNSUPPORTED  # 70000 grid rows
    assert call(Tq=0) == L.WALL_OK                            # empty: nothing launched


def test_fwd_gate_workspace_and_checks(lib):
    al = lambda x: (x + 255) // 256 * 256
    B, T, H, HQ, K, V = 2, 100, 4, 8, 64, 64
    fwd = lib.wall_attn_fwd_workspace(0, B, T, H, HQ, K, V, 0, 0)
    # the forward's layout, then the prefix scan's chunk carries: one fp32 row
    # of HQ*K per 32-row chunk, [B*ceil(T/32), HQ*K]
    assert lib.wall_attn_fwd_gate_workspace(0, B, T, H, HQ, K, V, 0, 0) == \
        fwd + al(4 * B * -(-T // 32) * HQ * K)
    # varlen (n_seq sequences packed in B*T = 100 rows): each may add a chunk
    assert lib.wall_attn_fwd_gate_workspace(0, 1, T, H, HQ, K, V, 0, 3) == \
        lib.wall_attn_fwd_workspace(0, 1, T, H, HQ, K, V, 0, 3) + al(4 * (-(-T // 32) + 3) * HQ * K)
    # fp32 (SIMT path): no anchored operands, no carries
    assert lib.wall_attn_fwd_gate_workspace(1, B, T, H, HQ, K, V, 0, 0) == \
        lib.wall_attn_fwd_workspace(1, B, T, H, HQ, K, V, 0, 0)
    need = lib.wall_attn_fwd_gate_workspace(0, B, T, H, HQ, K, V, 0, 0)

    def call(g=FAKE, P=FAKE, HQ=HQ, ws_bytes=need, dtype=0):
        return lib.wall_attn_fwd_gate(FAKE, FAKE, FAKE, g, dtype, B, T, H, HQ, K, V, 0.0, None,
                                      None, 0, None, 0, P, FAKE, FAKE, FAKE, ws_bytes, None)

    assert call(g=None) == L.WALL_ERR_INVALID_ARG
    assert call(P=None) == L.WALL_ERR_INVALID_ARG
    assert call(HQ=6) == L.WALL_ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == L.WALL_ERR_INVALID_ARG
    assert call(dtype=7) == L.WALL_ERR_INVALID_ARG


def test_timing_slot_mask(lib):
    # host-only: the mask selects slots; bits past the slot count are refused
    assert lib.wall_timing_enable_slots(1 << 4) == L.WALL_OK
    n = len(api.TIMING_SLOTS)
    assert lib.wall_timing_enable_slots(1 << (n - 1)) == L.WALL_OK
    assert lib.wall_timing_enable_slots(1 << n) == L.WALL_ERR_INVALID_ARG
    assert lib.wall_timing_enable_slots(0) == L.WALL_OK
    assert lib.wall_timing_enable(0) == L.WALL_OK


def test_prefix_rejects_bad_arguments(lib):
    pc = lib.wall_prefix_cumsum
    assert pc(FAKE, 3, FAKE, 1, 8, 4, 64, None, 0, None, None, None) == L.WALL_ERR_INVALID_ARG
    assert pc(None, 0, FAKE, 1, 8, 4, 64, None, 0, None, None, None) == L.WALL_ERR_INVALID_ARG
    assert pc(FAKE, 0, FAKE, 2, 8, 4, 64, FAKE, 1, None, None, None) == L.WALL_ERR_INVALID_ARG
    assert pc(FAKE, 0, FAKE, 1, 8, 1, 3, None, 0, None, None, None) == L.WALL_ERR_UNSUPPORTED


def test_workspace_sizes(lib):
    # backward: D, dq, dk^(h), dv^(h), two scalar-gate parts (+ its prefix);
    # the bf16 tensor-core path adds the anchored operands q^, k^ (bf16),
    # the 128-row block anchors (fp32) and one int flag per (sequence, head)
    B, T, HQ, K, V = 2, 100, 8, 64, 64
    rows = B * T
    al = lambda x: (x + 255) // 256 * 256
    simt = al(4 * rows * HQ) + 2 * al(4 * rows * HQ * K) + al(4 * rows * HQ * V) + \
        2 * al(4 * rows * HQ)
    nblk = B * ((T + 127) // 128)
    tc = 2 * al(2 * rows * HQ * K) + al(4 * nblk * HQ * K) + al(4 * B * HQ)

    assert lib.wall_attn_bwd_workspace(1, B, T, 4, HQ, K, V, 0, 0, 0) == simt        # fp32
    assert lib.wall_attn_bwd_workspace(1, B, T, 4, HQ, K, V, 1, 0, 0) == simt + al(4 * rows * HQ)
    # bf16 dense: the stored dS tiles (bf16 128 x 128) of every (b, h, I, J <= I)
    nb = (T + 127) // 128
    ds = al(B * HQ * nb * (nb + 1) // 2 * 128 * 128 * 2)
    assert lib.wall_attn_bwd_workspace(0, B, T, 4, HQ, K, V, 0, 0, 0) == simt + tc + ds
    # the least workspace: no dS tiles (the dq pass then recomputes them)
    assert lib.wall_attn_bwd_workspace_min(0, B, T, 4, HQ, K, V, 0, 0) == simt + tc
    # beyond 8 GiB of tiles (B=1, T=65536, HQ=16: 68.9 GB) none are kept
    Tb = 65536
    big = lib.wall_attn_bwd_workspace(0, 1, Tb, 4, HQ * 2, K, V, 0, 0, 0)
    simtb = al(4 * Tb * HQ * 2) + 2 * al(4 * Tb * HQ * 2 * K) + al(4 * Tb * HQ * 2 * V) + \
        2 * al(4 * Tb * HQ * 2)
    tcb = 2 * al(2 * Tb * HQ * 2 * K) + al(4 * (Tb // 128) * HQ * 2 * K) + al(4 * HQ * 2)
    assert big == simtb + tcb
    # varlen packing (B == 1, n_seq > 0): the lengths are on the device, so
    # the tiles of one sequence holding every block (ceil(T/128) + n_seq)
    simt1 = al(4 * T * HQ) + 2 * al(4 * T * HQ * K) + al(4 * T * HQ * V) + 2 * al(4 * T * HQ)
    tc1 = 2 * al(2 * T * HQ * K) + al(4 * ((T + 127) // 128 + 3) * HQ * K) + al(4 * 3 * HQ)
    nbv = (T + 127) // 128 + 3
    ds1 = al(HQ * nbv * (nbv + 1) // 2 * 128 * 128 * 2)
    assert lib.wall_attn_bwd_workspace(0, 1, T, 4, HQ, K, V, 0, 3, 0) == simt1 + tc1 + ds1
    # a window of 256 keys: a query block keeps itself and ceil(255/128) = 2
    # earlier key blocks: 1 + 2 + 3 + 3 + ... over nb = 8 blocks = 21 tiles
    Tw = 1000
    rw = B * Tw
    simtw = al(4 * rw * HQ) + 2 * al(4 * rw * HQ * K) + al(4 * rw * HQ * V) + 2 * al(4 * rw * HQ)
    tcw = 2 * al(2 * rw * HQ * K) + al(4 * B * 8 * HQ * K) + al(4 * B * HQ)
    assert lib.wall_attn_bwd_workspace(0, B, Tw, 4, HQ, K, V, 0, 0, 256) == \
        simtw + tcw + al(B * HQ * 21 * 128 * 128 * 2)
    assert lib.wall_attn_bwd_workspace(0, B, Tw, 4, HQ, K, V, 0, 0, 0) == \
        simtw + tcw + al(B * HQ * 36 * 128 * 128 * 2)
    assert lib.wall_attn_bwd_workspace(0, B, T, 4, HQ, 32, 32, 0, 0, 0) == \
        al(4 * rows * HQ) + 2 * al(4 * rows * HQ * 32) + al(4 * rows * HQ * 32) + \
        2 * al(4 * rows * HQ)                                                     # SIMT bf16
    assert lib.wall_attn_bwd_workspace(0, B, T, 3, HQ, K, V, 0, 0, 0) == 0           # bad shape
    assert lib.wall_attn_fwd_workspace(1, B, T, 4, HQ, K, V, 0, 0) == 0           # fp32, no opts
    assert lib.wall_attn_fwd_workspace(0, B, T, 4, HQ, K, V, 0, 0) == tc
    assert lib.wall_attn_decode_workspace(32, 32768, 8, 32, 128, 64) > 0
    assert lib.wall_attn_decode_workspace(1, 0, 1, 1, 64, 64) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "libwall.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(ImportError):
        L.lib()


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "channel_decay_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "wall_oracle" not in src, f


def test_library_errors_surface_as_wall_error(lib):
    """A status code from the library reaches Python as WallError, with the
    library's own description of it."""
    with pytest.raises(L.WallError, match="invalid argument") as e:
        L._check("wall_timing_enable_slots", lib.wall_timing_enable_slots(1 << 31))
    assert e.value.code == L.WALL_ERR_INVALID_ARG
    L._check("wall_timing_enable_slots", lib.wall_timing_enable_slots(0))
