"""The boundary from plain C: a C99 program that includes include/zb.h, links
against libzb.so and calls the entry points that touch no device
(zb_validate, zb_workspace_bytes, zb_merge_workspace_bytes,
zb_recalibrate_workspace_bytes, zb_strerror, zb_place_by_demand).  Checks
that the header is C (no C++ in it) and that its answers agree with the
Python binding's."""
import os
import subprocess

import numpy as np
import pytest

from token_dispatch_top_b200 import build, zb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <stdint.h>
#include "zb.h"

int main(void) {
  zb_config c = {0};
  c.P = 8; c.E = 64; c.K = 6; c.S = 4096; c.H = 2048; c.R = 2; c.C = 0.1f;
  c.gpus_per_node = 2; c.cap_rows = 4096 * 6; c.policy = ZB_POLICY_ROOM;
  c.relax = 0; c.repair = 0;
  printf("validate %d\n", zb_validate(&c));
  printf("ws %zu\n", zb_workspace_bytes(&c));
  printf("merge_ws %zu\n", zb_merge_workspace_bytes(&c));
  printf("recal_ws %zu %zu\n", zb_recalibrate_workspace_bytes(&c, 0),
         zb_recalibrate_workspace_bytes(&c, 1));
  printf("strerror %s\n", zb_strerror(ZB_ERR_CAPACITY));
  int64_t demand[64];
  for (int e = 0; e < 64; e++) demand[e] = (int64_t)(1000000 / (e + 1));
  int32_t pl[16];
  int st = zb_place_by_demand(&c, demand, pl);
  printf("place %d", st);
  for (int x = 0; x < 16; x++) printf(" %d", pl[x]);
  printf("\n");
  c.E = 65;  /* E % P != 0 */
  printf("invalid %d %zu\n", zb_validate(&c), zb_workspace_bytes(&c));
  return 0;
}
"""


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    build.build()
    d = tmp_path_factory.mktemp("c_consumer")
    src = d / "consumer.c"
    src.write_text(C_SOURCE)
    exe = d / "consumer"
    libdir = os.path.dirname(zb.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-l:libzb.so", f"-Wl,-rpath,{libdir}"])
    out = subprocess.check_output([str(exe)], text=True)
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


def test_header_is_c_and_answers_agree(program):
    cfg = zb.Config(P=8, E=64, K=6, S=4096, H=2048, R=2, C=0.1, gpus_per_node=2)
    assert int(program["validate"]) == zb.OK == zb.validate(cfg)
    assert int(program["ws"]) == zb.workspace_bytes(cfg) > 0
    lib = zb.load()
    import ctypes
    assert int(program["merge_ws"]) == lib.zb_merge_workspace_bytes(ctypes.byref(cfg.c())) > 0
    r0, r1 = (int(v) for v in program["recal_ws"].split())
    assert r0 == lib.zb_recalibrate_workspace_bytes(ctypes.byref(cfg.c()), 0) > 0
    assert r1 == lib.zb_recalibrate_workspace_bytes(ctypes.byref(cfg.c()), 1) > 0
    assert program["strerror"] == zb.strerror(zb.ERR_CAPACITY)
    st, *pl = (int(v) for v in program["place"].split())
    assert st == zb.OK
    demand = np.array([1000000 // (e + 1) for e in range(64)], np.int64)
    np.testing.assert_array_equal(np.array(pl).reshape(8, 2), zb.place_by_demand(cfg, demand))
    assert program["invalid"].split() == [str(zb.ERR_INVALID), "0"]
