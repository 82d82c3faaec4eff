"""The Python binding declares every C-ABI function with exactly the parameters
include/fapk.h gives it (a missing ctypes argtype passes a 64-bit pointer as a
C int)."""
import re
import os

from causal_flash_attention_packed_b200 import fapk

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fapk.h")


def test_argtypes_match_the_header():
    text = open(HEADER).read()
    decls = re.findall(r"FAPK_API\s+[\w\s\*]+?\b(fapk_\w+)\s*\(([^;]*?)\)\s*;", text, re.S)
    assert len(decls) >= 15
    L = fapk.lib()
    for name, params in decls:
        n = 0 if params.strip() in ("", "void") else len(params.split(","))
        argtypes = getattr(L, name).argtypes
        assert argtypes is not None, name
        assert len(argtypes) == n, (name, len(argtypes), n)
