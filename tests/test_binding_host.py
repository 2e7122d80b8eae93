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
    Top-k buffer, and the launch names / counts follow the grouping."""
    g = csa2.DecodeGroup(_cpu_cache(), ("F", "Ri", "Ri", "Ru", "Ru", "Ru"), 64, 512, 2048, concurrent=False)
    assert all(g.topk[layer] is g.topk[2] for layer in (3, 4, 5))
    assert len({id(g.topk[layer]) for layer in (0, 1, 2)}) == 3
    assert g.launch_names() == ["scan", "pool", "topk0", "attn0", "topk1", "attn1", "topk2", "attn2"]
    assert g.launches_per_step == len(g.launch_names())
    assert [w.numel() for w in g.attn_ws] == [csa2.attn_workspace_bytes(len(s), 1, 64) for s in g.sources]
    p = csa2.PrefillGroup(_cpu_cache(), 0, ("F", "Ru", "Ru", "Ru", "Ru", "Ru"), 16, 8, 64)
    assert all(t is p.topk[0] for t in p.topk)
    assert p.launch_names() == ["topk0", "attn0"] and p.launches_per_step == 3   # the indexer is two kernels
