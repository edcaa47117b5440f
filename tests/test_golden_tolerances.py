"""Our parity bar is at least as strict as the tolerances the pages state."""
import os

from tests.tolerances import OUT_MAX_ABS, OUT_REL_L2, STATE_REL_L2

HERE = os.path.dirname(os.path.abspath(__file__))


def _page_values():
    vals = {}
    for line in open(os.path.join(HERE, "golden", "page_tolerances.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_parity_bar_is_stricter_than_the_pages():
    v = _page_values()
    assert v == {"GDN_ATOL": 3e-2, "GDN_RTOL": 3e-2, "GDN_TREE_ATOL": 5e-2}
    assert OUT_MAX_ABS < v["GDN_ATOL"] and OUT_REL_L2 < v["GDN_RTOL"] and STATE_REL_L2 < v["GDN_RTOL"]
