"""avq_attention_noalloc: the attention call for callers that cannot allocate
device memory (a framework that owns all device allocations, or code that
cannot afford cudaMalloc's synchronisation), checked against avq_attention.

Both calls run the same kernels on the same inputs, so their outputs must be
identical bit for bit: any difference would be scratch left over from an
earlier call or a wrong scratch address.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test. It loads the library itself,
so it also passes alone in a fresh process.
"""
import pytest
import torch

from adaptive_vector_quantized_avq_b200 import binding as bd
from adaptive_vector_quantized_avq_b200 import build
from adaptive_vector_quantized_avq_b200 import synthetic as syn

import parity

pytestmark = pytest.mark.gpu

CASES = [
    # tensor-core kernel (bf16, tile 128): scratch = status word + value table
    syn.small_workload(B=2, H=3, N=1000, d=64, M0=64, C=4, tile=128, dtype="bf16", seed=31,
                       n_components=64, P=(8,)),
    syn.small_workload(B=1, H=2, N=700, d=128, M0=32, C=8, tile=128, dtype="bf16", seed=32,
                       n_components=40, P=(4,)),
    syn.WORKLOADS["vit-b"].with_(B=2),
    # CUDA-core kernel (fp32 inputs, or tile 64): no scratch, status cleared
    syn.small_workload(B=1, H=2, N=300, d=64, M0=16, C=4, tile=64, dtype="f32", seed=33,
                       n_components=16, P=(4,)),
    syn.small_workload(B=1, H=2, N=333, d=64, M0=32, C=4, tile=64, dtype="bf16", seed=34,
                       n_components=40, P=(6,)),
]


def _inputs(wl):
    inp = syn.generate(wl)
    K, V, Q, cb = (parity.to_device(getattr(inp, n), wl.dtype) for n in ("K", "V", "Q", "codebook"))
    _, counts, vsum = bd.precompute(K, V, cb, wl.M0, wl.C)
    return Q, cb, counts, vsum


def _noalloc(wl, Q, cb, counts, vsum, like_O, like_sel):
    shape = bd.make_shape(wl.B, wl.H, wl.N, wl.d, wl.M0, wl.C, Q.dtype)
    status = torch.full((1,), -99, dtype=torch.int32, device="cuda")
    O = torch.full_like(like_O, float("nan"))
    sel = torch.full_like(like_sel, -1)
    rc = bd.avq_attention_noalloc(shape, Q, cb, counts, vsum, wl.P[0], wl.tile, wl.softmax_scale, O, sel,
                                  status)
    assert rc == 0, bd.avq_status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return O, sel


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.dtype}-T{w.tile}-{w.B}x{w.H}x{w.N}x{w.d}-{w.M0}-{w.C}")
def test_noalloc_matches_workspace_call(wl):
    build.build()
    assert torch.cuda.is_available()
    Q, cb, counts, vsum = _inputs(wl)
    P = wl.P[0]
    O_ref, sel_ref = bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, wl.tile, wl.softmax_scale)
    torch.cuda.synchronize()
    for call in range(2):   # two calls in a row share (and reuse) the library's scratch
        O, sel = _noalloc(wl, Q, cb, counts, vsum, O_ref, sel_ref)
        assert torch.equal(sel, sel_ref), f"selection differs on call {call}"
        assert torch.equal(O, O_ref), \
            f"call {call}: O differs, max-abs {(O.float() - O_ref.float()).abs().max().item()}"


def test_noalloc_small_after_large():
    """A smaller problem right after a larger one: the scratch still holds the
    larger problem's value table, which the second call must not see."""
    build.build()
    big = syn.WORKLOADS["vit-b"].with_(B=2)
    small = syn.small_workload(B=1, H=2, N=520, d=64, M0=16, C=2, tile=128, dtype="bf16", seed=35,
                               n_components=16, P=(3,))
    for wl in (big, small):
        Q, cb, counts, vsum = _inputs(wl)
        P = wl.P[0]
        O_ref, sel_ref = bd.attention(Q, cb, counts, vsum, wl.M0, wl.C, P, wl.tile, wl.softmax_scale)
        torch.cuda.synchronize()
        O, sel = _noalloc(wl, Q, cb, counts, vsum, O_ref, sel_ref)
        assert torch.equal(sel, sel_ref) and torch.equal(O, O_ref), wl.name


def test_noalloc_rejects_oversized_problem():
    build.build()
    # scratch needed: 256 + B*H*M0*(1+C)*d*2 bytes > 8 MiB
    shape = bd.make_shape(64, 16, 128, 64, 128, 8, torch.bfloat16)
    fake = 1 << 40
    rc = bd.avq_attention_noalloc(shape, fake, fake, fake, fake, 4, 128, 0.125, fake, fake, None, 0)
    assert rc == -5, bd.avq_status_string(rc)   # AVQ_EWORKSPACE, nothing enqueued
