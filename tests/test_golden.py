"""Golden fixtures: the oracle against its committed snapshot, and the pages'
printed constants against the values the oracle tests use."""
import json
import os

import numpy as np

import oracle
from workloads import Spec, make_inputs, NAMED

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_snapshot():
    snap = json.load(open(os.path.join(HERE, "oracle_snapshot.json")))
    for case in snap["cases"]:
        sp = dict(case["spec"])
        if sp.get("grid") is not None:
            sp["grid"] = tuple(sp["grid"])
        spec = Spec(**sp)
        inp = make_inputs(spec, threads=1)
        o, st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin,
                                     spec.block_len, spec.eps)
        np.testing.assert_allclose(o.ravel(), case["out"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(st.ravel(), case["state"], rtol=1e-12, atol=1e-14)


def test_page_constants():
    pc = json.load(open(os.path.join(HERE, "page_constants.json")))
    assert pc["eps"]["value"] == 1e-8
    assert pc["head_dim"]["value"] == 32
    assert pc["head_dims_served"]["value"] == [32, 64]
    for spec in NAMED.values():
        assert spec.eps == pc["eps"]["value"]
        assert spec.d in pc["head_dims_served"]["value"]
        # the head count follows hidden_size // linear_head_dim at the model width of 2240
        if spec.d == 64:
            assert spec.H * spec.d == 2240
