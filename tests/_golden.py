"""Reader for the hand-derived fixtures under tests/golden/ (key = expression)."""
import math
import os
from fractions import Fraction

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name: str) -> dict:
    env = {"__builtins__": {}, "log": math.log, "exp": math.exp, "Fraction": Fraction}
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, expr = line.split("=", 1)
            out[key.strip()] = eval(expr.strip(), env)  # fixture expressions only
    return out
