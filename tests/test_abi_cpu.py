"""The C-ABI library loads on a machine without a GPU, exports every symbol
the header declares, and rejects bad arguments on the host before launching
anything. No compute calls are made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    from lightning_indexer_cross_b200 import build
    build.build()
    from lightning_indexer_cross_b200 import _abi
    return _abi


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "indexcache.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ic_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree(abi):
    assert _declared_symbols() == sorted(abi.EXPORTED)


def test_every_declared_symbol_is_exported(abi):
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(abi):
    for code in range(6):
        assert abi.ic_status_string(code).startswith("IC_")
    assert "unknown" in abi.ic_status_string(77)


def _fake(n=1 << 20):
    # host memory stands in for device pointers: validation must reject before any use
    buf = (ctypes.c_uint8 * n)()
    return ctypes.c_void_p(ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 256), buf


def test_indexer_rejects_bad_arguments(abi):
    p, keep = _fake()
    ws = p
    call = lambda **kw: abi._indexer(*[kw.get(n, d) for n, d in [
        ("q", p), ("w", p), ("k", p), ("ks", None), ("dt", abi.IC_BF16), ("B", 2), ("H", 64), ("d", 128),
        ("N", 1000), ("kbs", 0), ("sbs", 0), ("nv", None), ("s", p), ("ws", ws), ("wsb", 256), ("st", None)]])
    assert call(q=None) == abi.IC_ERR_INVALID_ARG
    assert call(B=0) == abi.IC_ERR_INVALID_ARG
    assert call(N=0) == abi.IC_ERR_INVALID_ARG
    assert call(d=96) == abi.IC_ERR_UNSUPPORTED
    assert call(H=129) == abi.IC_ERR_UNSUPPORTED
    assert call(dt=abi.IC_F32) == abi.IC_ERR_UNSUPPORTED
    assert call(dt=abi.IC_FP8_E4M3) == abi.IC_ERR_INVALID_ARG  # e4m3 keys need scales
    assert call(q=ctypes.c_void_p(p.value + 4)) == abi.IC_ERR_INVALID_ARG  # misaligned
    assert call(kbs=100) == abi.IC_ERR_INVALID_ARG  # stride shorter than a cache
    assert call(wsb=16) == abi.IC_ERR_INVALID_ARG
    assert call(ws=None) == abi.IC_ERR_INVALID_ARG


def test_topk_rejects_bad_arguments(abi):
    p, keep = _fake()
    call = lambda **kw: abi._topk(*[kw.get(n, d) for n, d in [
        ("s", p), ("B", 2), ("N", 1000), ("nv", None), ("k", 64), ("idx", p), ("ws", p), ("wsb", 1 << 20),
        ("st", None)]])
    assert call(k=0) == abi.IC_ERR_INVALID_ARG
    assert call(k=20000) == abi.IC_ERR_INVALID_ARG
    assert call(s=None) == abi.IC_ERR_INVALID_ARG
    assert call(wsb=300) == abi.IC_ERR_INVALID_ARG  # too small for the candidate buffers
    need = abi.ic_topk_workspace_size(2, 1000, 64)
    assert need >= 2 * 1000 * 8  # a candidate buffer (position, key) per row, here the whole row
    assert call(wsb=need - 256 - 1) == abi.IC_ERR_INVALID_ARG


def test_sparse_mla_rejects_bad_arguments(abi):
    p, keep = _fake()
    call = lambda **kw: abi._mla(*[kw.get(n, d) for n, d in [
        ("q", p), ("kv", p), ("kvs", 0), ("N", 100), ("idx", p), ("k", 16), ("sink", p), ("gate", None),
        ("sc", 0.04), ("B", 1), ("H", 8), ("od", abi.IC_BF16), ("out", p), ("lse", None), ("ws", p),
        ("wsb", 1 << 20), ("st", None)]])
    assert call(sc=0.0) == abi.IC_ERR_INVALID_ARG
    assert call(sc=-1.0) == abi.IC_ERR_INVALID_ARG
    assert call(sc=float("nan")) == abi.IC_ERR_INVALID_ARG
    assert call(od=abi.IC_FP8_E4M3) == abi.IC_ERR_UNSUPPORTED
    assert call(kvs=10) == abi.IC_ERR_INVALID_ARG
    assert call(sink=None) == abi.IC_ERR_INVALID_ARG
    assert call(wsb=64) == abi.IC_ERR_INVALID_ARG


def test_index_overlap_rejects_bad_arguments(abi):
    # every case fails on the host before any launch (the pointers are host memory)
    p, keep = _fake()
    call = lambda **kw: abi._overlap(*[kw.get(n, d) for n, d in [
        ("a", p), ("b", p), ("B", 2), ("k", 16), ("N", 100), ("count", p), ("st", None)]])
    assert call(a=None) == abi.IC_ERR_INVALID_ARG
    assert call(count=None) == abi.IC_ERR_INVALID_ARG
    assert call(B=0) == abi.IC_ERR_INVALID_ARG
    assert call(k=0) == abi.IC_ERR_INVALID_ARG
    assert call(N=0) == abi.IC_ERR_INVALID_ARG
    assert call(N=1851392 + 1) == abi.IC_ERR_UNSUPPORTED  # one bit per position in shared memory


def test_indexer_topk_rejects_bad_arguments(abi):
    # every case fails on the host before any launch (the pointers are host memory)
    p, keep = _fake()
    need = abi.ic_indexer_topk_workspace_size(2, 1000, 64, 0)
    assert 256 < need < (1 << 20)
    call = lambda **kw: abi._indexer_topk(*[kw.get(n, d) for n, d in [
        ("q", p), ("w", p), ("k", p), ("ks", None), ("dt", abi.IC_BF16), ("B", 2), ("H", 64), ("d", 128),
        ("N", 1000), ("kbs", 0), ("sbs", 0), ("nv", None), ("topk", 64), ("rpp", 0), ("idx", p), ("ws", p),
        ("wsb", need), ("st", None)]])
    assert call(q=None) == abi.IC_ERR_INVALID_ARG
    assert call(idx=None) == abi.IC_ERR_INVALID_ARG
    assert call(B=0) == abi.IC_ERR_INVALID_ARG
    assert call(topk=0) == abi.IC_ERR_INVALID_ARG
    assert call(ws=None) == abi.IC_ERR_INVALID_ARG
    assert call(wsb=need - 1) == abi.IC_ERR_INVALID_ARG  # one byte short of the score and top-k scratch
    # a pass of fewer rows needs less scratch
    assert abi.ic_indexer_topk_workspace_size(256, 264192, 2048, 128) < \
        abi.ic_indexer_topk_workspace_size(256, 264192, 2048, 0)


def test_topk_noalloc_rejects_bad_arguments(abi):
    p, keep = _fake()
    call = lambda **kw: abi._topk_noalloc(*[kw.get(n, d) for n, d in [
        ("s", p), ("B", 2), ("N", 1000), ("nv", None), ("k", 64), ("idx", p), ("st", None)]])
    assert call(s=None) == abi.IC_ERR_INVALID_ARG
    assert call(idx=None) == abi.IC_ERR_INVALID_ARG
    assert call(B=0) == abi.IC_ERR_INVALID_ARG
    assert call(N=0) == abi.IC_ERR_INVALID_ARG
    assert call(k=0) == abi.IC_ERR_INVALID_ARG
    assert call(k=16385) == abi.IC_ERR_INVALID_ARG
    assert call(B=abi.IC_TOPK_NOALLOC_MAX_ROWS + 1) == abi.IC_ERR_UNSUPPORTED


def test_context_parallel_steps_reject_bad_arguments(abi):
    p, keep = _fake()
    cand = lambda **kw: abi._cp_cand(*[kw.get(n, d) for n, d in [
        ("s", p), ("idx", p), ("B", 2), ("Nl", 1000), ("k", 64), ("off", 0), ("cs", p), ("ci", p), ("ws", p),
        ("wsb", 256), ("st", None)]])
    assert cand(ws=None) == abi.IC_ERR_INVALID_ARG
    assert cand(wsb=16) == abi.IC_ERR_INVALID_ARG
    assert cand(s=None) == abi.IC_ERR_INVALID_ARG
    assert cand(ci=None) == abi.IC_ERR_INVALID_ARG
    assert cand(B=0) == abi.IC_ERR_INVALID_ARG
    assert cand(k=0) == abi.IC_ERR_INVALID_ARG
    assert cand(Nl=0) == abi.IC_ERR_INVALID_ARG
    assert cand(off=-1) == abi.IC_ERR_INVALID_ARG
    assert cand(off=(1 << 31) - 500) == abi.IC_ERR_INVALID_ARG  # global positions past int32
    merge = lambda **kw: abi._cp_merge(*[kw.get(n, d) for n, d in [
        ("cs", p), ("ci", p), ("seg", 128), ("G", 2), ("B", 2), ("kin", 64), ("k", 64), ("lo", 0), ("hi", 1000),
        ("ig", p), ("il", None), ("st", None)]])
    assert merge(cs=None) == abi.IC_ERR_INVALID_ARG
    assert merge(ig=None) == abi.IC_ERR_INVALID_ARG
    assert merge(G=0) == abi.IC_ERR_INVALID_ARG
    assert merge(kin=0) == abi.IC_ERR_INVALID_ARG
    assert merge(lo=-1) == abi.IC_ERR_INVALID_ARG
    assert merge(lo=10, hi=5) == abi.IC_ERR_INVALID_ARG
    assert merge(seg=100) == abi.IC_ERR_INVALID_ARG  # segments overlap: B kin = 128 per rank
    assert merge(G=300) == abi.IC_ERR_UNSUPPORTED  # 300 x 64 candidates per row exceed shared memory
    rows = 2 * 8
    comb = lambda **kw: abi._cp_combine(*[kw.get(n, d) for n, d in [
        ("po", p), ("os", rows * 512), ("pl", p), ("ls", rows), ("G", 2), ("B", 2), ("H", 8), ("sink", p),
        ("gate", None), ("od", abi.IC_BF16), ("out", p), ("lse", None), ("st", None)]])
    assert comb(po=None) == abi.IC_ERR_INVALID_ARG
    assert comb(sink=None) == abi.IC_ERR_INVALID_ARG
    assert comb(out=None) == abi.IC_ERR_INVALID_ARG
    assert comb(G=0) == abi.IC_ERR_INVALID_ARG
    assert comb(od=abi.IC_FP8_E4M3) == abi.IC_ERR_UNSUPPORTED
    assert comb(po=ctypes.c_void_p(p.value + 4)) == abi.IC_ERR_INVALID_ARG  # misaligned
    assert comb(os=rows * 512 - 4) == abi.IC_ERR_INVALID_ARG  # segments overlap
    assert comb(os=rows * 512 + 1) == abi.IC_ERR_INVALID_ARG  # a segment off a 16-byte boundary
    assert comb(ls=rows - 1) == abi.IC_ERR_INVALID_ARG


def test_cache_append_rejects_bad_arguments(abi):
    # every case below must fail validation: the pointers are host memory
    p, keep = _fake()
    call = lambda **kw: abi._append(*[kw.get(n, d) for n, d in [
        ("kr", p), ("g", p), ("b", p), ("eps", 1e-6), ("dt", abi.IC_BF16), ("kc", p), ("ks", None), ("kbs", 0),
        ("sbs", 0), ("kvr", p), ("kvc", p), ("kvbs", 0), ("pos", p), ("T", 4), ("d", 128), ("N", 100),
        ("base", 10000.0), ("q", None), ("qp", None), ("B", 0), ("H", 0), ("ws", p), ("wsb", 256), ("st", None)]])
    assert call(kr=None) == abi.IC_ERR_INVALID_ARG
    assert call(pos=None) == abi.IC_ERR_INVALID_ARG
    assert call(T=0) == abi.IC_ERR_INVALID_ARG
    assert call(N=0) == abi.IC_ERR_INVALID_ARG
    assert call(d=96) == abi.IC_ERR_UNSUPPORTED
    assert call(dt=abi.IC_F32) == abi.IC_ERR_UNSUPPORTED
    assert call(dt=abi.IC_FP8_E4M3) == abi.IC_ERR_INVALID_ARG  # e4m3 keys need their scales
    assert call(ks=p) == abi.IC_ERR_INVALID_ARG                 # bf16 keys take none
    assert call(eps=-1.0) == abi.IC_ERR_INVALID_ARG
    assert call(eps=float("inf")) == abi.IC_ERR_INVALID_ARG
    assert call(base=0.0) == abi.IC_ERR_INVALID_ARG
    assert call(base=float("nan")) == abi.IC_ERR_INVALID_ARG
    assert call(kc=ctypes.c_void_p(p.value + 8)) == abi.IC_ERR_INVALID_ARG  # misaligned
    assert call(kbs=100 * 128 - 1) == abi.IC_ERR_INVALID_ARG   # caches would overlap
    assert call(kvbs=576) == abi.IC_ERR_INVALID_ARG
    assert call(q=p) == abi.IC_ERR_INVALID_ARG                  # q needs q_pos, B and H
    assert call(q=p, qp=p, B=2, H=0) == abi.IC_ERR_INVALID_ARG
    assert call(wsb=16) == abi.IC_ERR_INVALID_ARG
    assert call(ws=None) == abi.IC_ERR_INVALID_ARG
    assert abi.ic_cache_append_workspace_size() >= 4


def test_decompress_gate_rejects_bad_arguments(abi):
    # every case below must fail validation: the pointers are host memory
    p, keep = _fake()
    call = lambda **kw: abi._gate(*[kw.get(n, d) for n, d in [
        ("o", p), ("w", p), ("g", None), ("B", 4), ("H", 8), ("dv", 128), ("od", abi.IC_BF16), ("out", p),
        ("ws", p), ("wsb", 256), ("st", None)]])
    assert call(o=None) == abi.IC_ERR_INVALID_ARG
    assert call(out=None) == abi.IC_ERR_INVALID_ARG
    assert call(B=0) == abi.IC_ERR_INVALID_ARG
    assert call(H=0) == abi.IC_ERR_INVALID_ARG
    assert call(dv=64) == abi.IC_ERR_UNSUPPORTED
    assert call(od=abi.IC_FP8_E4M3) == abi.IC_ERR_UNSUPPORTED
    assert call(w=ctypes.c_void_p(p.value + 2)) == abi.IC_ERR_INVALID_ARG  # misaligned
    assert call(g=ctypes.c_void_p(p.value + 8)) == abi.IC_ERR_INVALID_ARG
    assert call(wsb=8) == abi.IC_ERR_INVALID_ARG
    assert abi.ic_decompress_gate_workspace_size() >= 4


@pytest.mark.parametrize("sched", [b"SFFF", b"FXSS", b"FS", b"FSSSS", b"", b"fsss"])
def test_stack_rejects_bad_schedules(abi, sched):
    p, keep = _fake()
    L = 4
    table = (abi.ic_layer_t * L)()
    for l in range(L):
        for f in ("q_idx", "w", "k_idx", "q", "kv", "sink", "out"):
            setattr(table[l], f, p.value)
    sh = abi.ic_stack_shape_t()
    sh.B, sh.N, sh.H_I, sh.d_I, sh.topk, sh.H, sh.sm_scale = 1, 4096, 4, 64, 256, 8, 0.04
    r = abi._stack(table, L, sched, ctypes.byref(sh), p, None, p, 1 << 20, None)
    assert r == abi.IC_ERR_INVALID_ARG


def test_stack_rejects_missing_indexer_inputs_on_f_layers(abi):
    p, keep = _fake()
    L = 3
    table = (abi.ic_layer_t * L)()
    for l in range(L):
        for f in ("q", "kv", "sink", "out"):
            setattr(table[l], f, p.value)
    table[0].q_idx, table[0].w, table[0].k_idx = p.value, p.value, p.value
    sh = abi.ic_stack_shape_t()
    sh.B, sh.N, sh.H_I, sh.d_I, sh.topk, sh.H, sh.sm_scale = 1, 4096, 4, 64, 256, 8, 0.04
    # layer 2 is F but has no indexer inputs
    assert abi._stack(table, L, b"FSF", ctypes.byref(sh), p, None, p, 1 << 30, None) == abi.IC_ERR_INVALID_ARG


def test_ops_refuse_cpu_tensors(abi):
    import torch
    from lightning_indexer_cross_b200 import ops
    q = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.indexer_score(q, torch.zeros(1, 4), torch.zeros(1, 10, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        ops.topk(torch.zeros(1, 10), 4)
    with pytest.raises(ValueError):
        ops.sparse_mla_decode(torch.zeros(1, 8, 576, dtype=torch.bfloat16),
                              torch.zeros(1, 10, 576, dtype=torch.bfloat16),
                              torch.zeros(1, 4, dtype=torch.int32), torch.zeros(8))
    with pytest.raises(ValueError):
        ops.cache_append(torch.zeros(2, 64, dtype=torch.bfloat16), torch.ones(64), torch.zeros(64),
                         torch.zeros(2, 576, dtype=torch.bfloat16), torch.zeros(2, dtype=torch.int64),
                         torch.zeros(1, 10, 64, dtype=torch.bfloat16), torch.zeros(1, 10, 576, dtype=torch.bfloat16))


def test_layer_struct_matches_header(abi):
    """ic_layer_t in the binding has the header's fields, in order."""
    text = open(os.path.join(ROOT, "include", "indexcache.h")).read()
    body = text[text.index("typedef struct {", text.index("ic_stack_shape_t;")):text.index("} ic_layer_t;")]
    names = re.findall(r"\*?\s*(\w+);", re.sub(r"/\*.*?\*/", "", body, flags=re.S))
    assert names == [f for f, _ in abi.ic_layer_t._fields_]
    assert ctypes.sizeof(abi.ic_layer_t) == 8 * len(names)
