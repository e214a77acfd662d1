"""The in-tree build rebuilds libattn.so whenever any file it is compiled from changes, so a stale
library can never be tested or timed: every source and header under csrc/ and the public header
are in its dependency list."""
import glob
import os

from exact_long_context_tmem_b200 import build as B


def test_every_csrc_file_is_a_dependency():
    deps = set(B.dependencies())
    files = glob.glob(os.path.join(B.CSRC, "*.cu")) + glob.glob(os.path.join(B.CSRC, "*.cuh")) + \
        glob.glob(os.path.join(B.CSRC, "*.cpp"))
    assert files
    for f in files:
        assert os.path.normpath(f) in deps, f
    assert os.path.normpath(os.path.join(B.ROOT, "include", "attn.h")) in deps


def test_edited_header_makes_library_stale(tmp_path, monkeypatch):
    """up_to_date compares modification times against every dependency, headers included."""
    lib = tmp_path / "libattn.so"
    lib.write_bytes(b"")
    monkeypatch.setattr(B, "LIB", str(lib))
    newest = max(os.path.getmtime(f) for f in B._inputs())
    os.utime(lib, (newest + 10, newest + 10))
    assert B.up_to_date()
    hdr = os.path.join(B.CSRC, "decode_int.cuh")
    os.utime(lib, (os.path.getmtime(hdr) - 10, os.path.getmtime(hdr) - 10))
    assert not B.up_to_date()
