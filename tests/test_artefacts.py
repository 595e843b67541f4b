"""The calibration artefact (per-layer thresholds saved once and loaded at
inference, Prox App. A.7): exact round trip and the checks on malformed files.
Host-only logic; no GPU needed."""

import json

import numpy as np
import pytest


@pytest.fixture(scope="module")
def art():
    from activation_sparse_swiglu_b200 import stack
    return stack


def test_round_trip_is_bit_exact(art):
    rng = np.random.default_rng(3)
    taus = [float(np.float32(v)) for v in rng.random(32) * 2]
    taus_s = [float(np.float32(v)) for v in rng.random(32) * 5]
    text = art.thresholds_to_json(taus, taus_s, d_model=4096, d_ff=14336, k=4301, s1=0.5, s2=0.7)
    doc = art.thresholds_from_json(text)
    assert [ly["tau_x"] for ly in doc["layers"]] == taus
    assert [ly["tau_s"] for ly in doc["layers"]] == taus_s
    for ly, t in zip(doc["layers"], taus):
        assert np.float32(ly["tau_x"]) == np.float32(t)
    doc2 = art.thresholds_from_json(art.thresholds_to_json(taus, d_model=4096, d_ff=14336, k=4301,
                                                           s1=0.5))
    assert all(ly["tau_s"] is None for ly in doc2["layers"]) and doc2["s2"] is None


def test_malformed_artefacts_are_refused(art):
    good = json.loads(art.thresholds_to_json([0.5, 0.6], [1.0, 2.0], d_model=512, d_ff=1376, k=413,
                                             s1=0.5, s2=0.7))
    bad_docs = []
    d = dict(good); d["format"] = "other"; bad_docs.append(d)
    d = dict(good); d["version"] = 99; bad_docs.append(d)
    d = dict(good); d["layers"] = []; bad_docs.append(d)
    d = dict(good); d["k"] = 0; bad_docs.append(d)
    d = json.loads(json.dumps(good)); d["layers"][0]["tau_x"] = -1.0; bad_docs.append(d)
    d = json.loads(json.dumps(good)); d["layers"][1]["tau_s"] = None; bad_docs.append(d)
    d = json.loads(json.dumps(good)); d["layers"][0]["tau_x"] = "0.5"; bad_docs.append(d)
    for doc in bad_docs:
        with pytest.raises(ValueError):
            art.thresholds_from_json(json.dumps(doc))
    with pytest.raises(ValueError):
        art.thresholds_from_json('{"format": "prox-thresholds", "version": 1, "d_model": 512,'
                                 ' "d_ff": 1376, "k": 413, "s1": 0.5, "s2": null,'
                                 ' "layers": [{"tau_x": NaN, "tau_s": null}]}')
    with pytest.raises(ValueError):
        art.thresholds_to_json([0.5], [1.0, 2.0], d_model=512, d_ff=1376, k=413, s1=0.5)
