"""CPU tests: the fp64 oracle against its pins, and the pins against planted
mistakes in the oracle."""
import pytest

from oracle import wall_oracle as wo
from tests import oracle_pins as pins


@pytest.fixture(autouse=True)
def _clean_oracle():
    wo.set_mutation(0)
    yield
    wo.set_mutation(0)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    ok, detail = pin()
    assert ok, detail


# Each planted mistake is a plausible oracle bug: a wrong product range, a
# dropped or sign-flipped term, a wrong head map or row index, an off-by-one
# window, a missing sink term, a misplaced scale and a wrong log base.
MUTATIONS = {
    1: "product over r=j..i",
    2: "key-side gate term dropped",
    3: "query-side gate term sign",
    4: "GQA head map h % H",
    5: "dv uses dO of the key row",
    6: "window i-j <= W",
    7: "sink left out of the normaliser",
    8: "scale on the scalar-gate bias",
    9: "prefix without 1/ln2",
}


@pytest.mark.parametrize("m", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_pins_catch_planted_mistake(m):
    wo.set_mutation(m)
    res = pins.run_all_pins()
    failed = [n for n, (ok, _) in res.items() if not ok]
    assert failed, f"mutation {m} ({MUTATIONS[m]}) passed every pin"
