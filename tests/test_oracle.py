"""The oracle against its pins, and the pins against planted mistakes (CPU only)."""
import os
import subprocess
import tempfile

import pytest

import oracle
import oracle_pins

PLANTS = {
    1: "rotation sign flipped",
    2: "sin and cos swapped",
    3: "half-split partner taken from the full head dim",
    4: "causal mask aligned top-left",
    5: "causal diagonal excluded",
    6: "softmax scale dropped",
    7: "max term dropped from lse",
    8: "kv head chosen modulo",
    9: "every query row rotated at position L",
    10: "v rows appended one row late",
    11: "rotary conjugate flag ignored",
    12: "left window one key short",
    13: "backward softmax Jacobian row term dropped",
    14: "backward scale missing from dk",
    15: "backward dk and dv from the group's last query head only",
}


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.load())


@pytest.fixture(scope="module")
def plant_dir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=lambda p: PLANTS[p].replace(" ", "-"))
def test_pins_catch_planted_mistake(plant, plant_dir):
    path = os.path.join(plant_dir, f"liboracle_plant{plant}.so")
    oracle.build(extra_flags=(f"-DORACLE_PLANT={plant}",), out_path=path)
    lib = oracle.load(path)
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {PLANTS[plant]}"
