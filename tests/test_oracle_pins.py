"""The CPU oracle against the facts that pin it (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS + [oracle_pins.pin_rejects_bad_shapes],
                         ids=lambda p: p.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_golden_file_parses():
    cases = oracle_pins.load_golden()
    assert [c["name"] for c in cases] == [
        "two_columns_one_row", "two_columns_two_rows", "three_columns",
        "four_columns", "one_column"]
    for c in cases:
        assert c["x"].shape == c["dout"].shape == c["out"].shape == c["dinp"].shape
