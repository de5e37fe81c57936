"""The entry point's smoke run (pack, GEMV, batched GEMV and a two-group stack on
cuda:0, each checked against the oracle) as a GPU test."""
import pytest


@pytest.mark.gpu
def test_smoke_entry_point():
    import __graft_entry__
    __graft_entry__.smoke()
