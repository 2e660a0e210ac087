"""The memory figures the pages print, recomputed with the oracle's helpers."""

import json
import os

import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "printed_memory_figures.json")
UNITS = {"GB": 1e9, "MB": 1e6, "KiB": 1024.0, "count": 1.0}


def _compute(fig):
    i = fig["inputs"]
    h = fig["helper"]
    if h == "naive_score_bytes":
        return oracle.naive_score_bytes(i["n"], i["heads"], i["elem_bytes"])
    if h == "flash_state_bytes":
        return oracle.flash_state_bytes(i["n"], i["d"], i["heads"], i["elem_bytes"])
    if h == "lse_bytes":
        return oracle.lse_bytes(i["n"], i["heads"])
    if h == "flash_state_bytes+lse_bytes":
        return oracle.flash_state_bytes(i["n"], i["d"], i["heads"], i["elem_bytes"]) + oracle.lse_bytes(i["n"], i["heads"])
    if h == "score_count":
        return oracle.score_count(i["n"])
    if h == "tile_bytes":
        return oracle.tile_bytes(i["rows"], i["cols"], i["elem_bytes"])
    raise KeyError(h)


FIGS = json.load(open(GOLDEN))["figures"]


@pytest.mark.parametrize("fig", FIGS, ids=[f["name"] for f in FIGS])
def test_printed_figure(fig):
    got = _compute(fig) / UNITS[fig["unit"]]
    if fig.get("at_least"):
        assert got > fig["value"]
    else:
        assert round(got, fig["digits"]) == pytest.approx(fig["value"]), (got, fig["printed"])
