"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import os
import re

import pytest

from adaptive_vector_quantized_avq_b200 import binding as bd
from adaptive_vector_quantized_avq_b200 import build as bl

HEADER = os.path.join(bl.ROOT, "include", "avq.h")


@pytest.fixture(scope="module")
def L():
    bl.build()
    return bd.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(avq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert set(names) == set(bd.EXPORTS), names
    for n in names:
        assert hasattr(L, n), f"{n} not exported"


def test_version_and_status_strings(L):
    assert bd.avq_version() >= 100
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert bd.avq_status_string(code).startswith(bd._STATUS[code])


def shape(**kw):
    a = dict(B=1, H=2, N=256, d=64, M0=16, C=4, dtype=bd.AVQ_BF16)
    a.update(kw)
    return bd.AvqShape(**a)


@pytest.mark.parametrize("bad", [dict(d=32), dict(d=96), dict(B=0), dict(H=0), dict(N=-1),
                                 dict(M0=0), dict(C=-1), dict(dtype=7), dict(M0=129), dict(C=0, M0=513)])
def test_workspace_query_rejects_bad_shapes(L, bad):
    assert bd.avq_precompute_workspace_bytes(shape(**bad)) == 0
    assert bd.avq_attention_workspace_bytes(shape(**bad), 2, 128) == 0


def test_workspace_sizes(L):
    s = shape()
    n = bd.avq_precompute_workspace_bytes(s)
    assert n >= 256 and n % 256 == 0
    m = bd.avq_attention_workspace_bytes(s, 4, 128)
    assert m >= 256 and m % 256 == 0
    assert bd.avq_attention_workspace_bytes(s, 17, 128) == 0    # P > M0
    assert bd.avq_attention_workspace_bytes(s, -1, 128) == 0
    assert bd.avq_attention_workspace_bytes(s, 4, 96) == 0      # tile not 64/128
    flat = shape(C=0, M0=512)                                    # a flat codebook of 512 codewords
    assert bd.avq_precompute_workspace_bytes(flat) >= 256
    assert bd.avq_attention_workspace_bytes(flat, 0, 128) >= 256 + 1 * 2 * 512 * 64 * 2
    assert bd.avq_attention_workspace_bytes(flat, 2, 128) == 0   # nothing to select
    assert bd.avq_attention_workspace_bytes(shape(C=0, M0=512, d=128), 0, 128) >= 256 + 2 * 512 * 128 * 2
    assert bd.avq_attention_workspace_bytes(shape(C=0, M0=512, d=128), 0, 64) == 0    # flat: tile 128 only


FAKE = 1 << 40   # 256-byte aligned, never dereferenced: validation fails first


def test_precompute_argument_errors(L):
    s = shape()
    ws = bd.avq_precompute_workspace_bytes(s)
    ok = dict(K=FAKE, V=FAKE, cb=FAKE, a=FAKE, c=FAKE, v=FAKE, w=FAKE)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return bd.avq_precompute(s if "s" not in kw else kw["s"], a["K"], a["V"], a["cb"], a["a"],
                                 a["c"], a["v"], a["w"], kw.get("wsb", ws), stream=0)

    assert call(K=0) == -1
    assert call(cb=0) == -1
    assert call(K=FAKE + 8) == -1             # misaligned (16 B rule)
    assert call(a=FAKE + 2) == -1             # misaligned (4 B rule)
    assert call(w=0) == -5
    assert call(wsb=ws - 1) == -5
    assert call(w=FAKE + 16) == -1            # workspace not 256-aligned
    assert call(s=shape(M0=129)) == -2
    assert call(s=shape(C=17)) == -2
    assert call(s=shape(d=80)) == -1


def test_attention_argument_errors(L):
    s = shape()
    ws = bd.avq_attention_workspace_bytes(s, 4, 128)

    def call(P=4, tile=128, scale=0.125, **kw):
        a = dict(Q=FAKE, cb=FAKE, c=FAKE, v=FAKE, O=FAKE, sel=FAKE, w=FAKE)
        a.update(kw)
        return bd.avq_attention(s, a["Q"], a["cb"], a["c"], a["v"], P, tile, scale, a["O"],
                                a["sel"], a["w"], kw.get("wsb", ws), stream=0)

    assert call(P=17) == -1
    assert call(P=-1) == -1
    assert call(tile=32) == -1
    assert call(scale=0.0) == -1
    assert call(scale=float("nan")) == -1
    assert call(Q=0) == -1
    assert call(sel=0) == -1
    assert call(O=FAKE + 4) == -1
    assert call(wsb=0) == -5


def test_flat_codebook_argument_rules(L):
    """C = 0: attention takes P = 0 only (nothing to select); the no-alloc entry
    point leaves flat codebooks to avq_attention; all decided on the host."""
    flat = shape(C=0, M0=256)
    ws = bd.avq_attention_workspace_bytes(flat, 0, 128)
    assert bd.avq_attention(flat, FAKE, FAKE, FAKE, FAKE, 2, 128, 0.125, FAKE, FAKE, FAKE, ws,
                            stream=0) == -1
    assert bd.avq_attention(flat, FAKE, FAKE, FAKE, FAKE, 0, 64, 0.125, FAKE, None, FAKE, ws,
                            stream=0) == -2   # flat attention takes tile 128 only
    assert bd.avq_attention_noalloc(flat, FAKE, FAKE, FAKE, FAKE, 0, 128, 0.125, FAKE, None,
                                    stream=0) == -2


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(bd, "_LIB", None)
    monkeypatch.setattr(bd, "library_path", lambda: str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        bd.lib()


def test_tensor_api_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 64)
    with pytest.raises(ValueError):
        bd.precompute(x, x, torch.zeros(1, 80, 64), 16, 4)


def test_deep_argument_errors(L):
    """Depth-L calls: depth, budgets and workspace are checked on the host."""
    s = shape(M0=16, C=4)
    ws = bd.avq_attention_deep_workspace_bytes(s, 3)
    assert ws == 256 + ((1 * 2 * 16 * (1 + 4 + 16) * 64 * 4 + 255) // 256) * 256   # status + fp32 means
    assert bd.avq_attention_deep_workspace_bytes(s, 1) == 0
    assert bd.avq_attention_deep_workspace_bytes(s, 5) == 0

    def att(P=(4, 8), Lv=3, tile=128, wsb=None, **kw):
        a = dict(Q=FAKE, cb=FAKE, c=FAKE, v=FAKE, O=FAKE, sel=FAKE, w=FAKE)
        a.update(kw)
        return bd.avq_attention_deep(s, Lv, P, a["Q"], a["cb"], a["c"], a["v"], tile, 0.125, a["O"], a["sel"],
                                     a["w"], ws if wsb is None else wsb, stream=0)

    assert att(Lv=1, P=()) == -1
    assert att(Lv=5, P=(1, 1, 1, 1)) == -1
    assert att(P=(17, 8)) == -1        # more than the 16 level-0 nodes
    assert att(P=(4, 17)) == -1        # more than the 4 * 4 level-1 candidates
    assert att(P=(4, 33)) == -1        # 33 * 4 > 128 slots
    assert att(P=(-1, 0)) == -1
    assert att(tile=32) == -1
    assert att(sel=0) == -1
    assert att(wsb=0) == -5
    assert bd.avq_precompute_deep(s, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0) == -1
    assert bd.avq_precompute_deep(shape(M0=129, C=2), 3, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, stream=0) == -2
    assert bd.avq_precompute_deep(s, 3, FAKE, 0, FAKE, FAKE, FAKE, FAKE, stream=0) == -1
