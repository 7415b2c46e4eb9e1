"""The C-ABI library loads without a GPU and exports every entry point that
include/lsq.h declares; its host-side NF4 codebook equals the oracle's bit for
bit (the two are computed by separate code from the same definition)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lsq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(lsq_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    from nf4_layer_streamed_blockwise_b200 import lib
    declared = _declared()
    assert len(declared) >= 20
    missing = [n for n in declared if n not in lib.exported_symbols()]
    assert not missing, f"declared in include/lsq.h but not exported: {missing}"
    bound = set(lib._SIGS)
    assert set(declared) <= bound, f"not bound in lib.py: {set(declared) - bound}"


def test_status_strings_and_version():
    from nf4_layer_streamed_blockwise_b200 import lib
    assert lib.lsq_version() >= 100
    assert lib.lsq_status_str(0) == "ok"
    assert "page-locked" in lib.lsq_status_str(2)


def test_codebook_bitexact_with_oracle():
    from nf4_layer_streamed_blockwise_b200 import lib
    from oracle import nf4
    got = np.array(lib.lsq_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), nf4.codebook().view(np.uint32))
