"""The build entry point's smoke run (one tiny causal forward + backward on cuda:0 against the
oracle) passes."""

import pytest

pytestmark = pytest.mark.gpu


def test_smoke():
    import __graft_entry__
    __graft_entry__.smoke()
