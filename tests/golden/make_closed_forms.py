"""Writes closed_forms.json: values fixed by mathematics, used as pins.

* ln_V: the loss of a uniform prediction over V tokens (all-zero LM head),
  natural log as in the pages' cross-entropy (reading notes §2.2).
* window_pairs: sum_{t=1}^{T} min(t, k) of eq. (1) for the full-size
  workloads, from the oracle's direct summation.

Run: python tests/golden/make_closed_forms.py
"""
import json
import math
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import window_pairs  # noqa: E402

out = {
    "source": "ln V: natural-log CE of a uniform distribution; window_pairs: eq. (1) of the reading notes",
    "ln_V": {str(V): math.log(V) for V in (64, 1024, 128256)},
    "window_pairs": {f"{T},{k}": window_pairs(T, k) for T, k in ((4096, 1024), (8192, 8192), (32768, 8192), (131072, 8192))},
}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.json"), "w") as fh:
    json.dump(out, fh, indent=1)
print(json.dumps(out, indent=1))
