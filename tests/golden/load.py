"""Readers for the page-cited fixtures in this folder."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def e2m1_codepoints():
    with open(os.path.join(HERE, "e2m1_codepoints.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                return [float(t) for t in line.split()]
    raise ValueError("no code points")


def format_facts():
    out = {}
    with open(os.path.join(HERE, "format_facts.txt")) as f:
        for line in f:
            line = line.split("|")[0].strip()
            if not line or line.startswith("#"):
                continue
            k, v = (t.strip() for t in line.split("="))
            out[k] = float(v)
    return out
