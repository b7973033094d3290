"""loopkv_append_noalloc against loopkv_append, through the C ABI.

loopkv_append_noalloc serves callers that cannot allocate device memory (an engine whose own
arena already holds the device's memory, or a decode loop that cannot take the device-wide
synchronisation an allocation may cause): it stages the batch's request ids in a fixed array
inside the library instead of the cache's staging words.  Two caches built from the same plan
and history take the same appends, one through each entry point, twice in a row; their tails
and tail lengths must be equal bit for bit, and decodes of both within the parity tolerance.
This file is collected last so that a run stopping at the first failure has run every other
test before it.
"""
import pytest
import torch

from mixed_precision_kv_append_b200 import loopkv as L
from mixed_precision_kv_append_b200 import synth

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3


def _pair():
    modes = [L.CELL_4B, L.CELL_SHARE, L.CELL_2B, L.CELL_4B]  # 2 layers x 2 loops
    w = synth.Workload("noalloc", 2, 2, 4, 128, 5, [40, 64, 7, 96, 33], torch.bfloat16, modes, 0.01, seed=21)
    caches = []
    plan = L.Plan(w.n_layers, w.n_loops, w.H, w.D, w.B, w.max_blocks, w.modes, w.tau, w.tau_mode, w.dtype)
    for _ in range(2):
        c = L.Cache(plan)
        for layer in range(w.n_layers):
            for req in range(w.B):
                ks, vs = synth.layer_history(w, layer, req, device="cuda")
                for lp in range(w.n_loops):
                    c.ingest(lp, layer, req, ks[lp].contiguous(), vs[lp].contiguous())
        c.check("ingest")
        caches.append(c)
    return w, plan, caches


def test_noalloc_append_matches_append_twice():
    w, plan, (ref, new) = _pair()
    batches = [[3, 0, 4], [1, 2, 0, 4, 3]]  # two calls in a row, different sizes and orders
    for call, ids in enumerate(batches):
        _, ks, vs = synth.step_tokens(w, call, 0, device="cuda")
        for layer in range(w.n_layers):
            for lp in range(w.n_loops):
                k = ks[lp][: len(ids)].contiguous()
                v = vs[lp][: len(ids)].contiguous()
                L.loopkv_append(ref.handle, lp, layer, k, v, req_ids=ids)
                L.loopkv_append_noalloc(new.handle, lp, layer, k, v, req_ids=ids)
        torch.cuda.synchronize()
        ref.check(f"append call {call}")
        new.check(f"noalloc call {call}")
        for layer in range(w.n_layers):
            for lp in range(w.n_loops):
                h_ref, t_ref = ref.lengths(lp, layer)
                h_new, t_new = new.lengths(lp, layer)
                assert torch.equal(h_ref, h_new) and torch.equal(t_ref, t_new)
                for req in range(w.B):
                    n = int(t_ref[req])  # slots past the tail length hold whatever the buffer held
                    assert torch.equal(ref.tail(lp, layer, req)[:, :, :n], new.tail(lp, layer, req)[:, :, :n]), \
                        (call, lp, layer, req)
                q = synth.step_tokens(w, 7 + call, layer, device="cuda")[0][lp].contiguous()
                o_ref = ref.decode(lp, layer, q)
                o_new = new.decode(lp, layer, q)
                assert float((o_ref - o_new).abs().max()) <= OUT_ATOL
        ref.check("decode")
        new.check("decode")


def test_noalloc_append_rejects_oversized_batches():
    plan = L.Plan(1, 1, 1, 64, L.NOALLOC_MAX_IDS + 1, 2, [L.CELL_4B], 0.0)
    cache = L.Cache(plan)
    B = L.NOALLOC_MAX_IDS + 1
    k = torch.zeros((B, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LoopKVError) as e:
        L.loopkv_append_noalloc(cache.handle, 0, 0, k, k, req_ids=list(range(B)))
    assert e.value.code == -2
    # at the maximum the call goes through
    kk = k[: L.NOALLOC_MAX_IDS].contiguous()
    L.loopkv_append_noalloc(cache.handle, 0, 0, kk, kk, req_ids=list(range(L.NOALLOC_MAX_IDS))[::-1])
    cache.check("append at the maximum")
    _, tail = cache.lengths(0, 0)
    assert int(tail[: L.NOALLOC_MAX_IDS].sum()) == L.NOALLOC_MAX_IDS and int(tail[B - 1]) == 0
