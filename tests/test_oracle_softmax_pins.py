"""The fp64 softmax / top-K oracle against its pins, and planted mistakes against the
pins (each mistake lives only in a copy of the oracle's source, on the CPU)."""
import os
import types

import pytest

from oracle import softmax as osm
from tests import pin_softmax

SRC = osm.__file__


@pytest.mark.parametrize("name", sorted(pin_softmax.PINS))
def test_softmax_oracle_pin(name):
    pin_softmax.PINS[name](osm)


MUTANTS = {
    "max_not_subtracted": ("e = np.exp(a - m)", "e = np.exp(a)"),
    "max_sign_flipped": ("e = np.exp(a - m)", "e = np.exp(m - a)"),
    "not_normalised": ("return e / d, (m + np.log(d))[:, 0]", "return e, (m + np.log(d))[:, 0]"),
    "lse_without_max": ("return e / d, (m + np.log(d))[:, 0]", "return e / d, np.log(d)[:, 0]"),
    "min_for_max": ("m = a.max(axis=1, keepdims=True)", "m = a.min(axis=1, keepdims=True)"),
    "topk_ascending": ("order = np.lexsort((cols, -a[r]))", "order = np.lexsort((cols, a[r]))"),
    "topk_ties_to_higher_index": ("order = np.lexsort((cols, -a[r]))", "order = np.lexsort((-cols, -a[r]))"),
    "topk_off_by_one": ("idx[r] = order[:k]", "idx[r] = order[1:k + 1] if k < V else order[:k]"),
    "topk_probs_of_input": ("probs = np.take_along_axis(y, idx, axis=1)",
                            "probs = np.take_along_axis(np.exp(a), idx, axis=1)"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType("oracle_softmax_mutant")
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_softmax_mistake_fails_a_pin(name):
    import numpy as np
    with np.errstate(all="ignore"):
        assert pin_softmax.failures(_mutant(name)), f"planted mistake {name!r} passed every pin"
