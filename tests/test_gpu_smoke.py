"""The entry point's smoke check (one tiny round on cuda:0 against the oracle) as a GPU test,
so a change that breaks it shows in the suite."""
import pytest

import __graft_entry__

pytestmark = pytest.mark.gpu


def test_smoke_round_matches_oracle():
    __graft_entry__.smoke()
