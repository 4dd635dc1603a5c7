"""Expert cache on the GPU: outputs through the HBM slots equal the all-resident
layer bit for bit, the copy trace replays exactly in the oracle LRU, and the
host-side fault injections leave the cache unchanged."""
import numpy as np
import pytest
import torch

import expert_ffn_layer_route_b200 as moe
import moe_inputs as mi
from expert_ffn_layer_route_b200.offload import OffloadedBank
from oracle.lru import replay

pytestmark = pytest.mark.gpu

STAT_KEYS = ("lookups", "hits", "misses", "evictions", "prefetch_issued", "prefetch_used")


def _bank(shape, L, C, T, seed=0):
    bank = OffloadedBank(shape, L, C, T)
    layers = []
    for l in range(L):
        lay = mi.bank_layer(shape, l, seed, "cuda")
        bank.fill_layer(l, lay)
        layers.append(lay)
    return bank, layers


def _direct(shape, lay, x):
    desc = moe.make_desc(shape, x.shape[0])
    ws = torch.empty(moe.moe_workspace_size(desc), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(x)
    moe.moe_layer_forward(desc, x, lay["router"], lay["bias"], moe.make_weights(lay["experts"]), None, out, ws)
    return out


@pytest.mark.parametrize("fmt,C", [("nvfp4", 5), ("mxfp4", 12), ("int4", 7)])
def test_cache_outputs_equal_resident_layer_and_trace_replays(fmt, C):
    shape = mi.BANK.replace(d_model=512, d_ff=384 if fmt != "int4" else 256, n_experts=16, top_k=4, wdtype=fmt)
    L, T = 3, 4
    bank, layers = _bank(shape, L, C, T)
    bank.prefetch_top = shape.top_k  # prefetch every predicted expert (the driver's default is none)
    for step in range(3):
        x0 = mi.bank_step_tokens(step, T, shape.d_model, 5, "cuda")
        _, ins, outs = bank.decode_step(x0, prefetch=True, keep=True)
        torch.cuda.synchronize()
        for l in range(L):
            ref = _direct(shape, layers[l], ins[l])
            assert torch.equal(outs[l], ref), (step, l)
    assert moe.moe_get_last_error() == 0
    st = bank.stats()
    r = replay(bank.trace, L, shape.n_experts, C)
    assert {k: st[k] for k in STAT_KEYS} == r.stats
    for l in range(L):
        assert bank.cache.slot_map(l) == r.slot_map(l)
    assert st["prefetch_issued"] > 0
    copies = st["misses"] + st["prefetch_issued"]
    assert st["bytes_h2d"] == copies * bank.blob.size
    assert st["copy_ms"] > 0.0
    bank.close()


def test_injected_copy_failure_leaves_cache_unchanged(monkeypatch):
    monkeypatch.setenv("MOE_FAULT_INJECT", "copy")
    cache = moe.ExpertCache(2, 8, 3, 4096, device=0)
    sm = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        cache.lookup(0, [1, 2], sm)
    assert err.value.status == 7
    assert cache.slot_map(0) == [-1] * 8
    assert cache.stats()["lookups"] == 0
    cache.lookup(0, [1, 2], sm)  # the injection fires once
    torch.cuda.synchronize()
    assert cache.slot_map(0)[1:3] == [0, 1]
    assert sm.cpu().tolist()[1:3] == [0, 1]
    cache.close()


def test_injected_host_alloc_failure(monkeypatch):
    monkeypatch.setenv("MOE_FAULT_INJECT", "host_alloc")
    with pytest.raises(moe.MoeError) as err:
        moe.ExpertCache(2, 8, 3, 4096, device=0)
    assert err.value.status == 7


def test_full_size_bank_layer_through_cache():
    """One offloaded-bank layer at its real size (d=4096, 256 NVFP4 experts,
    64 slots) against the all-resident layer, two steps."""
    shape = mi.BANK
    bank, layers = _bank(shape, 1, mi.BANK_SLOTS_PER_LAYER, 16)
    for step in range(2):
        x0 = mi.bank_step_tokens(step, 16, shape.d_model, 9, "cuda")
        _, ins, outs = bank.decode_step(x0, prefetch=False, keep=True)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], _direct(shape, layers[0], ins[0]))
    bank.close()
