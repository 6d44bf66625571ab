"""CPU pins of the oracle (see ``pins.py`` for what each one checks and why)."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL, ids=lambda c: getattr(c, "__name__", None)
                         or c.func.__name__ + "_wd")
def test_pin(oracle_lib, check):
    check()
