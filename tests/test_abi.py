"""The C-ABI library loads and exports every entry point include/*.h declares;
host-only parts (status strings, workspace sizes, argument validation, which
returns before anything touches the GPU) behave as documented.  No GPU needed.
"""
import ctypes
import glob
import os
import re

import pytest

import eagle_tree_verification_dynamic_b200 as et
from eagle_tree_verification_dynamic_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        for m in re.finditer(r"EAGLE_API\s+[\w\s\*]+?\b(eagle_\w+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    return et.lib()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(_lib.exported_names())


def test_status_strings_and_version(lib):
    assert lib.eagle_status_string(0) == b"ok"
    assert lib.eagle_status_string(4) == b"size exceeds a library limit"
    assert lib.eagle_status_string(99) == b"unknown status"
    assert lib.eagle_version() >= 100


def test_workspace_sizes_are_pure_and_aligned(lib):
    a = lib.eagle_tree_build_workspace_bytes(4, 41, 128256, 1, 8)
    assert a > 0 and a % 256 == 0
    assert a == lib.eagle_tree_build_workspace_bytes(4, 41, 128256, 1, 8)
    assert lib.eagle_tree_attention_workspace_bytes(1, 60, 32, 32, 128, 2048, 0) > 0
    assert lib.eagle_accept_workspace_bytes(32, 32, 128256, 1) > 0
    assert lib.eagle_row_stats_workspace_bytes(0, 10, 0, 1) == 0      # invalid -> 0
    assert lib.eagle_tree_build_workspace_bytes(1, 5, 1000, 7, 2) == 0  # bad dtype -> 0


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first


def _tree(valid=True):
    p = FAKE if valid else None
    return _lib.TreeStruct(p, p, p, p, None, p, p)


def test_build_validation(lib):
    st = _tree()
    n = ctypes.c_int(0)
    call = lambda **kw: lib.eagle_tree_build(
        kw.get("x", FAKE), kw.get("dt", 0), kw.get("B", 1), kw.get("R", 5), kw.get("V", 1000),
        kw.get("depth", 3), kw.get("k", 2), kw.get("m", 10), ctypes.byref(kw.get("tree", st)),
        ctypes.byref(n), kw.get("ws", FAKE), kw.get("wsb", 0), None)
    assert call(x=None) == 1
    assert call(tree=_tree(False)) == 1
    assert call(dt=5) == 3
    assert call(B=0) == 2
    assert call(R=6) == 2                        # R must be 1 + (depth-1) k
    assert call(k=33, R=1 + 2 * 33) == 4         # k > EAGLE_MAX_TOPK
    assert call(m=129) == 4
    assert call(depth=17, R=1 + 16 * 2) == 4
    assert call(depth=16, k=32, R=1 + 15 * 32) == 4   # pool > EAGLE_MAX_POOL
    assert call(k=1001, V=1000, R=1 + 2 * 1001) == 4  # k > V
    assert call(ws=None, wsb=0) == 5             # workspace required
    assert call(ws=ctypes.c_void_p(0x1001), wsb=1 << 30) == 5  # misaligned workspace


def test_attention_validation(lib):
    def call(**kw):
        return lib.eagle_tree_attention(
            kw.get("q", FAKE), FAKE, FAKE, FAKE, 128, FAKE, FAKE, FAKE, kw.get("pos", None), 1,
            kw.get("n", 10), kw.get("Hq", 4), kw.get("Hkv", 4), kw.get("D", 64), kw.get("window", 0), 0.0,
            kw.get("out", FAKE), FAKE, 1 << 30, None)
    assert call(q=None) == 1
    assert call(window=16, pos=None) == 1
    assert call(Hq=6, Hkv=4) == 2
    assert call(D=96) == 4
    assert call(n=129) == 4
    assert call(q=ctypes.c_void_p(0x1008)) == 6   # not 16-byte aligned


def test_accept_and_mask_validation(lib):
    def acc(**kw):
        return lib.eagle_accept(FAKE, kw.get("dt", 0), kw.get("draft", None), 0, kw.get("lse", None), 5,
                                FAKE, FAKE, FAKE, kw.get("u", None), 1, kw.get("n", 10), 1000,
                                kw.get("depth", 3), FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert acc(u=FAKE) == 1                      # sampling needs the draft logits and lse
    assert acc(u=FAKE, draft=FAKE) == 1
    assert acc(dt=9) == 3
    assert acc(n=200) == 4
    assert acc(depth=0) == 2
    rule = lambda r: lib.eagle_accept_with_rule(FAKE, 0, FAKE, 0, FAKE, 5, FAKE, FAKE, FAKE, FAKE, r, 1, 10, 1000, 3,
                                                FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert rule(2) == 2 and rule(-1) == 2
    assert lib.eagle_accept_with_rule(FAKE, 0, None, 0, None, 5, FAKE, FAKE, FAKE, FAKE, 1, 1, 10, 1000, 3,
                                      FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.eagle_tree_mask(None, None, None, 1, 10, FAKE, None, None) == 1
    assert lib.eagle_tree_mask(FAKE, None, None, 1, 129, FAKE, None, None) == 4
    assert lib.eagle_tree_mask(FAKE, None, None, 1, 10, FAKE, FAKE, None) == 1  # pos needs depth, prefix_len


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(et.EagleError):
        et.tree_build(torch.zeros(1, 5, 100), 3, 2, 10)


def _step_in(**kw):
    d = dict(draft_logits=FAKE, target_logits=FAKE, logits_dtype=0, B=1, V=32000, depth=6, k=10, m=60,
             q=FAKE, k_cache=FAKE, v_cache=FAKE, prefix_len=FAKE, Lmax=2048, k_tree=FAKE, v_tree=FAKE,
             Hq=32, Hkv=32, D=128, window=0, scale=0.0, uniforms=None, sampling_rule=0, block_table=None,
             page_size=0, pages_per_seq=0, num_pages=0)
    d.update(kw)
    return _lib.StepIn(*[d[name] for name, _ in _lib.StepIn._fields_])


def _step_out(valid=True):
    p = FAKE if valid else None
    return _lib.StepOut(_tree(), p, p, p, p, p, p)


def test_step_workspace_covers_the_four_calls(lib):
    si = _step_in()
    total = lib.eagle_verify_step_workspace_bytes(ctypes.byref(si))
    assert total > 0 and total % 256 == 0
    parts = (lib.eagle_tree_build_workspace_bytes(1, 51, 32000, 0, 10)
             + lib.eagle_tree_attention_workspace_bytes(1, 60, 32, 32, 128, 2048, 0)
             + lib.eagle_accept_workspace_bytes(1, 60, 32000, 0))
    assert parts <= total <= parts + 3 * 256
    off = lib.eagle_verify_step_attention_status_offset(ctypes.byref(si))
    assert off % 256 == 0 and off >= lib.eagle_tree_build_workspace_bytes(1, 51, 32000, 0, 10)
    assert lib.eagle_verify_step_workspace_bytes(ctypes.byref(_step_in(D=0))) == 0


def test_step_validation(lib):
    n = ctypes.c_int(0)

    def call(si=None, so=None, ws=FAKE, wsb=1 << 30):
        si = si or _step_in()
        so = so or _step_out()
        return lib.eagle_verify_step(ctypes.byref(si), ctypes.byref(so), ctypes.byref(n), ws, wsb, None)
    assert lib.eagle_verify_step(None, None, None, FAKE, 0, None) == 1
    assert call(si=_step_in(q=None)) == 1
    assert call(so=_step_out(False)) == 1
    assert call(si=_step_in(logits_dtype=4)) == 3
    assert call(si=_step_in(Hq=30, Hkv=4)) == 2
    assert call(si=_step_in(D=96)) == 4
    assert call(si=_step_in(m=200)) == 4
    assert call(si=_step_in(q=ctypes.c_void_p(0x1008))) == 6
    assert call(ws=None, wsb=0) == 5
    assert call(si=_step_in(sampling_rule=2)) == 2
    assert call(si=_step_in(block_table=FAKE, page_size=48, pages_per_seq=40, num_pages=100)) == 2
    assert call(si=_step_in(block_table=FAKE, page_size=64, pages_per_seq=40, num_pages=100), ws=None, wsb=0) == 5
    paged = lib.eagle_verify_step_workspace_bytes(ctypes.byref(_step_in(block_table=FAKE, page_size=64,
                                                                         pages_per_seq=32, num_pages=100, Lmax=0)))
    assert paged == lib.eagle_verify_step_workspace_bytes(ctypes.byref(_step_in(Lmax=2048)))
    assert n.value == 0  # nothing was reported: every call above failed validation


def test_kv_compact_validation(lib):
    def call(**kw):
        return lib.eagle_kv_compact(kw.get("kt", FAKE), FAKE, FAKE, FAKE, kw.get("plen", FAKE), FAKE, FAKE,
                                    kw.get("out", ctypes.c_void_p(0x2000)), 1, kw.get("n", 10), 8,
                                    kw.get("D", 128), 2048, kw.get("depth", 6), None)
    assert call(kt=None) == 1
    assert call(D=100) == 2                                   # D % 8 != 0
    assert call(plen=ctypes.c_void_p(0x2000)) == 2           # in-place length update is refused
    assert call(n=129) == 4
    assert call(depth=17) == 4
    assert call(kt=ctypes.c_void_p(0x1008)) == 6


def test_tree_grow_validation(lib):
    nb = lib.eagle_tree_grow_state_bytes(2, 32000, 0, 6, 10)
    assert nb > 0 and nb % 256 == 0
    assert lib.eagle_tree_grow_state_bytes(2, 32000, 5, 6, 10) == 0
    begin = lambda **kw: lib.eagle_tree_grow_begin(kw.get("x", FAKE), kw.get("dt", 0), 2, 32000, kw.get("depth", 6),
                                                   kw.get("k", 10), kw.get("st", FAKE), kw.get("nb", nb), None, None,
                                                   None)
    assert begin(x=None) == 1
    assert begin(dt=3) == 3
    assert begin(k=33) == 4
    assert begin(nb=nb - 1) == 5
    assert begin(st=ctypes.c_void_p(0x1010)) == 5              # state not 256-byte aligned
    lvl = lambda level: lib.eagle_tree_grow_level(FAKE, 0, 2, 32000, 6, 10, level, FAKE, nb, None, None, None)
    assert lvl(1) == 2 and lvl(7) == 2
    n = ctypes.c_int(0)
    fin = lambda levels, m, t: lib.eagle_tree_grow_finish(0, 2, 32000, 6, 10, levels, m, FAKE, nb, t,
                                                         ctypes.byref(n), None)
    assert fin(6, 60, None) == 1
    assert fin(6, 129, ctypes.byref(_tree())) == 4
    assert fin(0, 60, ctypes.byref(_tree())) == 2 and fin(7, 60, ctypes.byref(_tree())) == 2
    assert lib.eagle_tree_grow_gains(0, 2, 32000, 6, 10, FAKE, nb, None, None) == 1


def test_static_tree_validation(lib):
    arr = lambda v: (ctypes.c_int32 * len(v))(*v)
    par, rk = arr([0, 0, 1, 1, 3]), arr([0, 1, 0, 1, 0])
    assert lib.eagle_static_tree_rows(par, rk, 5) == 3
    assert lib.eagle_static_tree_rows(arr([0, 2]), arr([0, 0]), 2) == -1      # parent after its child
    assert lib.eagle_static_tree_rows(arr([0, 0]), arr([1, 1]), 2) == -1      # two siblings, one rank
    assert lib.eagle_static_tree_rows(arr([0]), arr([32]), 1) == -1           # rank beyond the top-k limit
    assert lib.eagle_static_tree_rows(par, rk, 0) == -1
    nb = lib.eagle_static_tree_workspace_bytes(4, 1000, 1, par, rk, 5)
    assert nb > 0 and nb % 256 == 0
    assert lib.eagle_static_tree_workspace_bytes(4, 1000, 1, arr([0, 2]), arr([0, 0]), 2) == 0
    t = _tree()
    build = lambda **kw: lib.eagle_static_tree_build(kw.get("x", FAKE), 0, 4, kw.get("R", 3), kw.get("V", 1000),
                                                     kw.get("par", par), rk, 5, ctypes.byref(t), FAKE,
                                                     kw.get("nb", nb), None)
    assert build(x=None) == 1
    assert build(R=4) == 2
    assert build(par=arr([0, 0, 1, 1, 5])) == 2
    assert build(V=1) == 4                                                     # rank 1 needs two tokens
    assert build(nb=nb - 1) == 5


def test_paged_validation(lib):
    FAKE2 = ctypes.c_void_p(0x2000)
    def att(**kw):
        d = dict(num_pages=100, ps=64, bt=FAKE, pps=8, B=2, n=10, Hq=32, Hkv=8, D=128, window=0, ws=FAKE,
                 nb=1 << 30)
        d.update(kw)
        return lib.eagle_tree_attention_paged(FAKE, FAKE, FAKE, d["num_pages"], d["ps"], d["bt"], d["pps"], FAKE, FAKE,
                                              FAKE, FAKE, FAKE, d["B"], d["n"], d["Hq"], d["Hkv"], d["D"], d["window"],
                                              0.0, FAKE, d["ws"], d["nb"], None)
    assert att(bt=None) == 1
    assert att(ps=48) == 2 and att(ps=8) == 2 and att(ps=0) == 2
    assert att(ps=192, nb=16) == 5                # a multiple of 64 passes; the short workspace stops the call
    assert att(num_pages=1 << 20, ps=4096) == 4   # pool rows past int range
    assert att(D=96) == 4
    assert att(ws=None, nb=0) == 5
    comp = lambda **kw: lib.eagle_kv_compact_paged(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("np", 100),
                                                   kw.get("ps", 16), kw.get("bt", FAKE), 8, kw.get("nl", FAKE2), 2,
                                                   10, 8, 128, 6, None)
    assert comp(bt=None) == 1 and comp(ps=24) == 2 and comp(nl=FAKE) == 2   # new lengths aliasing prefix_len
