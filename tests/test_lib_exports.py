"""The C-ABI library builds for sm_100a and exports every entry point that
include/*.h declares (CPU only: nothing is called on a device)."""

import ctypes
import glob
import os
import re

import pytest

from lossless_draft_verify_vc_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"VC_API\s+[\w\s\*]+?\b(vc_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def libpath():
    return B.build()


def test_header_declares_entry_points():
    names = _declared()
    for must in ["vc_draft_attn_quant", "vc_draft_attn_sparse", "vc_verify_attn", "vc_accept"]:
        assert must in names


def test_every_declared_symbol_is_exported(libpath):
    lib = ctypes.CDLL(libpath)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_error_text(libpath):
    lib = ctypes.CDLL(libpath)
    lib.vc_abi_version.restype = ctypes.c_int
    src = open(os.path.join(ROOT, "include", "vc.h")).read()
    want = int(re.search(r"#define VC_ABI_VERSION (\d+)", src).group(1))
    assert lib.vc_abi_version() == want
    lib.vc_last_error.restype = ctypes.c_char_p
    assert isinstance(lib.vc_last_error(), bytes)
