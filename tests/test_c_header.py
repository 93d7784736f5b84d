"""The boundary from C: a C11 program (not C++) includes include/longspark.h with every
warning as an error, links liblongspark.so and calls the host-side queries, which need no
GPU. Its answers must equal the Python binding's."""

import os
import shutil
import subprocess

import pytest

import fixed_cost_drafter_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stddef.h>
#include <stdio.h>
#include "longspark.h"

int main(void) {
  ls_config c = {0};
  c.batch = 16; c.n_layers = 4; c.n_kv_heads = 8; c.n_q_heads = 32; c.head_dim = 128;
  c.hidden = 4096; c.block = 16; c.window = 512; c.n_scales = 3;
  c.scales[0] = 64; c.scales[1] = 512; c.scales[2] = 4096;
  c.slots_per_scale = 32; c.dtype = LS_BF16; c.flags = 0;
  ls_layout y;
  const int st = ls_get_layout(&c, &y);
  ls_config bad = c;
  bad.window = 4;  /* < B + 1 */
  ls_layout y2;
  printf("%d %zu %zu %zu %zu %d %d %zu %d %s\n", st, ls_state_bytes(&c), y.total_bytes, y.off_kv,
         y.off_prologue, y.kv_rows, ls_get_layout(&bad, &y2), ls_view_state_bytes(&c, LS_VIEW_WINDOW),
         ls_get_layout(NULL, &y2), ls_status_string(LS_ERR_SHAPE));
  /* struct layouts the binding mirrors */
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(ls_config), offsetof(ls_config, scales),
         offsetof(ls_config, flags), sizeof(ls_layout), offsetof(ls_layout, kv_rows),
         offsetof(ls_layout, off_sample), offsetof(ls_layout, off_prologue), sizeof(ls_paged_kv),
         offsetof(ls_paged_kv, page_stride), offsetof(ls_paged_kv, block_table), offsetof(ls_paged_kv, num_pages),
         offsetof(ls_paged_kv, verify_slots));
  return 0;
}
"""


def test_header_compiles_as_c_and_links(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(F.library_path())
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, str(src), "-o", str(exe), "-L", libdir, "-llongspark",
                    "-Wl,-rpath," + libdir], check=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    out = lines[0].split()
    cfg = F.make_config(batch=16, n_layers=4, n_kv_heads=8, n_q_heads=32, head_dim=128, hidden=4096, block=16,
                        window=512, scales=[64, 512, 4096], slots_per_scale=32, dtype=F.LS_BF16)
    y = F.ls_get_layout(cfg)
    assert int(out[0]) == F.LS_OK
    assert int(out[1]) == int(out[2]) == F.ls_state_bytes(cfg) == y.total_bytes
    assert int(out[3]) == y.off_kv and int(out[4]) == y.off_prologue and int(out[5]) == y.kv_rows
    assert int(out[6]) == F.LS_ERR_SHAPE
    assert int(out[7]) == F.ls_view_state_bytes(cfg, F.LS_VIEW_WINDOW)
    assert int(out[8]) == F.LS_ERR_INVALID_ARG
    assert " ".join(out[9:]) == F.ls_status_string(F.LS_ERR_SHAPE)
    # the ctypes mirrors of the header's structs: same size, same field offsets
    import ctypes
    sz = [int(v) for v in lines[1].split()]
    C, Y, P = F.ls_config, F.ls_layout, F.ls_paged_kv
    assert sz == [ctypes.sizeof(C), C.scales.offset, C.flags.offset, ctypes.sizeof(Y), Y.kv_rows.offset,
                  Y.off_sample.offset, Y.off_prologue.offset, ctypes.sizeof(P), P.page_stride.offset,
                  P.block_table.offset, P.num_pages.offset, P.verify_slots.offset]
