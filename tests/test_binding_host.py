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
