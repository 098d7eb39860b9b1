"""Writes the stored expected values under tests/golden/ by calling only the oracle.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def worked_example():
    # Inputs printed by "Attention Kernel", section "Blockwise reference":
    # scores [1, -inf, 3, -2, 0], values arange(15) viewed as 5 x 3, block size 2;
    # the page asserts the result equals softmax(score) @ value, and that an
    # all -inf row gives zeros(3).
    score = [1.0, float("-inf"), 3.0, -2.0, 0.0]
    value = np.arange(15, dtype=np.float64).reshape(5, 3)
    o, lse = oracle.softmax_attend(score, value)
    o2, lse2 = oracle.online_attend(score, value, 2)
    assert np.allclose(o, o2, rtol=0, atol=1e-12)
    return {
        "source": "Attention Kernel, section 'Blockwise reference' (worked example)",
        "score": ["-inf" if s == float("-inf") else s for s in score],
        "value_shape": [5, 3],
        "value": value.reshape(-1).tolist(),
        "block_size": 2,
        "expected_o": [float(x) for x in o],
        "expected_lse": float(lse),
        "all_masked_expected_o": [0.0, 0.0, 0.0],
        "written_by": "tests/golden/make_golden.py (oracle only)",
    }


if __name__ == "__main__":
    path = os.path.join(HERE, "worked_example.json")
    with open(path, "w") as f:
        json.dump(worked_example(), f, indent=1)
        f.write("\n")
    print("wrote", path)
