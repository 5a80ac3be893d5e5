"""The boundary as a C program sees it: tests/c_abi/abi_consumer.c includes include/cowa.h as
strict C99 (-Wall -Wextra -Werror -pedantic), links libcowa.so and calls the host-side entry
points; its visible counts and tile plans must equal the oracle's (bit-exact), and the compute
entry points must return each documented status for bad arguments before any launch.  No GPU is
used."""

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import cowa_oracle as orc
from structured_sparse_attention_cowa_b200 import cowa as cw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "structured_sparse_attention_cowa_b200")


@pytest.fixture(scope="module")
def consumer_output(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    cw.lib()  # raises if libcowa.so has not been built
    exe = str(tmp_path_factory.mktemp("cabi") / "abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "abi_consumer.c"), "-L", PKG, "-lcowa",
                    f"-Wl,-rpath,{PKG}", "-o", exe], check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    lines = [ln.split() for ln in run.stdout.splitlines()]
    return lines


def _values(lines, key):
    return [ln[1:] for ln in lines if ln[0] == key]


def test_counts_and_plans_from_c_match_the_oracle(consumer_output):
    op = orc.Pattern(S=4, L=6, T=64, D=4)
    want = orc.visible_counts(70, op, 4)
    got = np.array([[int(x) for x in row[1:]] for row in sorted(_values(consumer_output, "counts"),
                                                                   key=lambda r: int(r[0]))])
    assert np.array_equal(got, want)
    fwd = sorted(tuple(int(x) for x in r) for r in _values(consumer_output, "fwd_plan"))
    want_f = sorted((g, i, j, int(full)) for (i, g), lst in orc.tile_plan_fwd(70, 32, 16, op, 4).items()
                    for j, full in lst)
    assert fwd == want_f
    bwd = sorted(tuple(int(x) for x in r) for r in _values(consumer_output, "bwd_plan"))
    want_b = sorted((g, j, i, 0) for (j, g), lst in orc.tile_plan_bwd(70, 32, 16, op, 4).items() for i in lst)
    assert bwd == want_b


def test_statuses_from_c(consumer_output):
    v = {ln[0]: ln[1:] for ln in consumer_output}
    assert v["version"] == ["1"]
    assert v["compact_rows"] == ["20736"]
    assert v["fwd_workspace"] == ["256"]
    assert {k: int(v[k][0]) for k in ("err_null_pattern", "err_head_dim", "err_group", "err_align",
                                       "err_workspace", "err_pattern", "err_tp_range")} == {
        "err_null_pattern": 1, "err_head_dim": 2, "err_group": 1, "err_align": 3, "err_workspace": 4,
        "err_pattern": 1, "err_tp_range": 1}
    strings = {int(r[0]): " ".join(r[1:]) for r in _values(consumer_output, "status")}
    assert sorted(strings) == list(range(7)) and strings[0] == "ok"
    assert len(set(strings.values())) == 7
