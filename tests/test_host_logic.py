"""Host-side logic of the binding that needs no GPU."""
import pytest

from block_sparse_attention_aware_b200 import fvattn


@pytest.mark.parametrize("H,want", [(40, 20), (4, 2), (2, 1), (1, 1), (3, 1), (6, 3), (9, 3), (7, 1), (12, 6)])
def test_default_head_groups(H, want):
    groups = fvattn.default_head_groups(H)
    assert groups == want
    assert H % groups == 0
    assert groups == 1 or H // groups >= 2
