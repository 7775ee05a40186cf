"""The in-tree build tracks every header its sources include: an edit to any
of them must rebuild the library and every cached object."""
import glob
import os

from selective_state_space_40_b200 import build as b


def test_every_header_keys_the_build():
    files = [p for p in glob.glob(os.path.join(b.CSRC, "*")) if os.path.isfile(p) and not p.endswith(".cu")]
    files += glob.glob(os.path.join(b.INCLUDE, "*"))
    assert files, "no headers found"
    assert set(files) <= set(b.headers())
