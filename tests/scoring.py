"""The pass rule of the dataset card "wan2.2_production_values", section
"Scoring / loss (the rule)", restated: a candidate output passes against a
reference iff every element is finite, the smallest per-(batch, head) cosine
over the flattened (S, D) slice is at least 0.9999, and the absolute
difference has max <= 3e-2 and mean <= 1e-4 (the card casts both sides with
``.float()``).  The thresholds live in tests/golden/scoring_rule.json; the
comparison itself is tests/common.py.
"""
from __future__ import annotations

import json
import os

_RULE = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scoring_rule.json")))
MIN_COS = _RULE["min_head_cosine"]
MAX_ABS = _RULE["max_abs_diff"]
MEAN_ABS = _RULE["mean_abs_diff"]
