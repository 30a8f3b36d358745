"""The debug build (libzo_b200_debug.so, ZO_DEBUG): device bounds checks that record a bit
of a device word and skip the access, never trap.

* On valid input the checks change nothing: probe steps (fp32 and bf16 tensor cores, across
  a lazy-window boundary), a generation query and the tensor-core attention op give the same
  bits as the release library, and no check fires.
* A planted bad index is caught: with ZO_DEBUG_PLANT=attention_tile the debug build's
  zo_op_attention points its last work tile at a row past the batch.  The kernel reads
  nothing for that tile (its rows keep the caller's fill), reports bit 0 of the word, and
  every other output row is the release library's bit for bit.

Each run is a child process (tests/debug_scenario.py) with its own library.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from gpu_util import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SCENARIO = os.path.join(HERE, "debug_scenario.py")


def _debug_lib():
    path = os.path.join(ROOT, "zeroth_order_fine_b200", "libzo_b200_debug.so")
    if not os.path.exists(path):
        from zeroth_order_fine_b200 import build
        build.build(debug=True)
    return path


def _run(args, debug, plant=None):
    env = dict(os.environ)
    env.pop("ZO_LIB", None)
    env.pop("ZO_DEBUG_PLANT", None)
    if debug:
        env["ZO_LIB"] = "debug"
    if plant:
        env["ZO_DEBUG_PLANT"] = plant
    r = subprocess.run([sys.executable, SCENARIO] + args, cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_checks_change_no_bit_and_do_not_fire_on_valid_input(tmp_path):
    _debug_lib()
    rel = _run(["model"], debug=False)
    dbg = _run(["model"], debug=True)
    assert rel.pop("debug_build") == 0 and dbg.pop("debug_build") == 1
    assert rel.pop("debug_word") == 0
    assert dbg.pop("debug_word") == 0
    assert rel == dbg
    (tmp_path / "r").mkdir()
    (tmp_path / "d").mkdir()
    ra = _run(["attention", str(tmp_path / "r")], debug=False)
    da = _run(["attention", str(tmp_path / "d")], debug=True)
    assert da["debug_word"] == 0 and ra["attention"] == da["attention"]


def test_planted_attention_tile_is_caught_and_skipped(tmp_path):
    sys.path.insert(0, HERE)
    import debug_scenario as ds
    _debug_lib()
    (tmp_path / "r").mkdir()
    (tmp_path / "p").mkdir()
    _run(["attention", str(tmp_path / "r")], debug=False)
    p = _run(["attention", str(tmp_path / "p")], debug=True, plant="attention_tile")
    assert p["debug_word"] & 1, p
    ref = np.load(tmp_path / "r" / "attention.npy")
    got = np.load(tmp_path / "p" / "attention.npy")
    last = sum(ds.ATTN_LENS[:-1])                  # the last row: its only tile was planted
    assert np.all(got[last:] == 7.0)               # nothing written there
    assert np.array_equal(got[:last], ref[:last])  # every other row as in the release build
    assert not np.all(ref[last:] == 7.0)
