"""The package's smoke entry point (one small prefill, its backward and a decode
step on cuda:0, each checked against the fp64 oracle) runs clean."""
import os
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_smoke_entry_point():
    sys.path.insert(0, ROOT)
    try:
        import __graft_entry__
    finally:
        sys.path.remove(ROOT)
    __graft_entry__.smoke()
