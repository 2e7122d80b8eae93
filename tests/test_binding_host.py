"""Host logic of the binding that needs no GPU: how a layer group's layers
share Top-k (and so attention launches)."""
import pytest

from kv_cache_decode_index_b200 import csa2


@pytest.mark.parametrize("modes,want", [
    (("F", "Ri", "Ri", "Ru", "Ru", "Ru"), [[0], [1], [2, 3, 4, 5]]),     # decoder group 1F+2Ri+3Ru
    (("F", "Ri", "Ri", "Ri", "Ri", "Ru"), [[0], [1], [2], [3], [4, 5]]),  # decoder group 1F+4Ri+1Ru
    (("F", "Ru", "Ru", "Ru", "Ru", "Ru"), [[0, 1, 2, 3, 4, 5]]),          # encoder group 1F+5Ru
    (("F",), [[0]]),
    (("Ri", "Ru"), [[0, 1]]),
])
def test_layer_sources(modes, want):
    assert csa2.layer_sources(modes) == want


@pytest.mark.parametrize("modes", [(), ("Ru", "F"), ("F", "X")])
def test_layer_sources_rejects(modes):
    with pytest.raises(ValueError):
        csa2.layer_sources(modes)


def _cpu_cache():
    import numpy as np
    return csa2.Cache(4, 128, np.arange(4, dtype=np.int32)[None, :], [500], device="cpu")


def test_groups_alias_reuse_topk_and_count_launches():
    """Built on host tensors (no launch): Reuse layers share their source's
    Top-k buffer; with a pool the step is scan, pool, one two-kernel Top-k of
    every index layer and one attention launch; without one, one flat Top-k
    per index layer."""
    g = csa2.DecodeGroup(_cpu_cache(), ("F", "Ri", "Ri", "Ru", "Ru", "Ru"), 64, 512, 2048)
    assert all(g.topk[layer] is g.topk[2] for layer in (3, 4, 5))
    assert len({id(g.topk[layer]) for layer in (0, 1, 2)}) == 3
    assert g.index_layers == [0, 1, 2]
    assert g.launch_names() == ["scan", "pool", "topk", "attn"] and g.launches_per_step == 5
    assert g.attn_ws.numel() == csa2.attn_workspace_bytes(6, 1, 64)
    assert g.rs_ws.numel() == csa2.reindex_layers_workspace_bytes(1, 3, 2048)
    assert g.hist.shape == (1, csa2.POOL_HIST_BINS) and int(g.hist.abs().sum()) == 0
    assert int(g.rs_ws.sum()) == 0    # the histograms start at zero
    g2 = csa2.DecodeGroup(_cpu_cache(), ("F", "Ri", "Ri", "Ri", "Ri", "Ru"), 64, 512, None)
    assert g2.launch_names() == ["scan", "topk", "attn"] and g2.launches_per_step == 2 + 5
    assert g2.hist is None and g2.pool is None
    p = csa2.PrefillGroup(_cpu_cache(), 0, ("F", "Ru", "Ru", "Ru", "Ru", "Ru"), 16, 8, 64)
    assert all(t is p.topk[0] for t in p.topk)
    assert p.launch_names() == ["topk0", "attn0"] and p.launches_per_step == 3   # the indexer is two kernels
