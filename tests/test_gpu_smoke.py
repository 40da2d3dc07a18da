"""The GPU smoke entry point (one tiny greedy generation through the C ABI, checked against
the oracle) runs green."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__ as entry
    entry.smoke()
