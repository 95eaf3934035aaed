"""Loads the hand-worked cases in tests/golden/hand_cases.json as numpy inputs."""

import json
import os

import numpy as np

import synth

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.json")


def _val(x):
    return -np.inf if x == "-inf" else float(x)


def cases():
    with open(_PATH) as f:
        doc = json.load(f)
    out = []
    for c in doc["cases"]:
        q = np.array(c["q"], dtype=np.float32)
        kc = np.array(c["kc"], dtype=np.float32)
        w = np.array(c["w"], dtype=np.float32)
        out.append({
            "name": c["name"],
            "m": c["m"],
            "k": c["k"],
            "q": synth.f32_to_bf16_bits(q),
            "kc": synth.f32_to_bf16_bits(kc),
            "w": w,
            "idx": np.array(c["idx"], dtype=np.int32),
            "score": np.array([[_val(v) for v in row] for row in c["score"]], dtype=np.float64),
        })
    return out
