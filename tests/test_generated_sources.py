"""Generated kernel sources match their generators: csrc/tmem_ops.inc is exactly what
csrc/gen_tmem_ops.py renders (so the committed wrappers can be regenerated from the
tree), and every wrapper it declares is one of the widths the kernels use."""

import importlib.util
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "sequence_approximate_attention_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_tmem_ops", os.path.join(CSRC, "gen_tmem_ops.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_tmem_ops_inc_is_generated():
    committed = open(os.path.join(CSRC, "tmem_ops.inc")).read()
    assert _gen().render() == committed


def test_tmem_wrappers_cover_the_widths_in_use():
    gen = _gen()
    used = set()
    for name in os.listdir(CSRC):
        if name.endswith((".cuh", ".cu")):
            used |= set(re.findall(r"tmem_(ld|st)_x(\d+)(_async)?\(", open(os.path.join(CSRC, name)).read()))
    for kind, n, asy in used:
        widths = gen.ASYNC_STORE_WIDTHS if asy else gen.LOAD_WIDTHS if kind == "ld" else gen.STORE_WIDTHS
        assert int(n) in widths, (kind, n, asy)
