"""The entry point's smoke check (one small decode step in the multi-kernel
and the cluster step, compared with the oracle) runs on the GPU too."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke():
    import __graft_entry__ as entry
    entry.smoke()
