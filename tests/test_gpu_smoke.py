"""The entry point's smoke check (one small forward + backward against the
oracle on cuda:0) runs to completion."""
import pytest

pytestmark = pytest.mark.gpu


def test_graft_entry_smoke():
    import __graft_entry__
    __graft_entry__.smoke()
