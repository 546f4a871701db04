"""Reader for the small hand-written fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    """Parse ``key: v1 v2 ...`` lines; '#' starts a comment.  Keys ending in
    ``_rowN`` are stacked into a 2-D array under the stem."""
    fields, rows = {}, {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = line.split(":", 1)
            vals = [float(v) for v in val.split()]
            if "_row" in key:
                stem, r = key.rsplit("_row", 1)
                rows.setdefault(stem, {})[int(r)] = vals
            else:
                fields[key.strip()] = np.array(vals)
    for stem, d in rows.items():
        fields[stem] = np.array([d[i] for i in sorted(d)])
    return fields
