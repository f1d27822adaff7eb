"""The entry point's smoke check (one small run of every kernel family
against the oracle) runs as part of the GPU suite."""
import pytest

pytestmark = pytest.mark.gpu


def test_graft_entry_smoke():
    import __graft_entry__

    __graft_entry__.smoke()
