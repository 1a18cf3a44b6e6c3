"""The C-ABI library loads, exports every entry point include/ls.h declares, its
argument structs match the ctypes mirrors byte for byte, and host-side argument
checks answer before anything touches a device.  CPU only."""
import ctypes as C
import os
import re
import subprocess
import tempfile

import pytest

from sparse_attention_decode_ls_b200 import binding as B
from sparse_attention_decode_ls_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ls.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ls_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["ls_index_score", "ls_topk_select", "ls_block_bound_prune", "ls_hotbuf_resolve",
              "ls_gather_misses", "ls_sparse_attn_decode", "ls_decode_step", "ls_get_error_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ls_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_version(lib):
    assert "sm_100a" in B.version()


def _c_layout(struct_name, fields):
    src = ["#include <stdio.h>", "#include <stddef.h>", f'#include "{HEADER}"', "int main(void) {",
           f'  printf("%zu\\n", sizeof({struct_name}));']
    for f in fields:
        src.append(f'  printf("%zu\\n", offsetof({struct_name}, {f}));')
    src += ["  return 0;", "}"]
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write("\n".join(src))
        subprocess.run(["gcc", "-std=c11", c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    return vals[0], vals[1:]


@pytest.mark.parametrize("name", sorted(B.STRUCTS))
def test_struct_layout_matches_header(name):
    st = B.STRUCTS[name]
    fields = [f for f, _ in st._fields_]
    size, offs = _c_layout(name, fields)
    assert C.sizeof(st) == size
    assert [getattr(st, f).offset for f in fields] == offs


def _err(lib, status):
    assert status != B.LS_OK
    assert lib.ls_get_error_string().decode() != ""
    return status


def test_host_checks_reject_bad_arguments(lib):
    # NULL struct
    assert _err(lib, lib.ls_index_score(None, None)) == B.LS_ERR_INVALID_ARG
    assert _err(lib, lib.ls_topk_select(None, None)) == B.LS_ERR_INVALID_ARG
    # top-k: k out of range, misaligned stride
    t = B.TopkArgs(batch=1, k=5000, max_len=64, scores=16, lens=16, idx=16)
    assert _err(lib, lib.ls_topk_select(C.byref(t), None)) == B.LS_ERR_INVALID_ARG
    t = B.TopkArgs(batch=1, k=8, max_len=63, scores=16, lens=16, idx=16)
    assert _err(lib, lib.ls_topk_select(C.byref(t), None)) == B.LS_ERR_INVALID_ARG
    # indexer: unsupported e4m3 shape, missing scales, null pointer
    a = B.IndexScoreArgs(batch=1, heads=32, dim=128, max_pages=1, max_len=64, key_dtype=B.LS_E4M3,
                         w_dtype=B.LS_BF16, num_pages=1, q=16, q_scale=16, w=16, key_pool=16, key_scale=16,
                         page_table=16, lens=16, scores=16)
    assert _err(lib, lib.ls_index_score(C.byref(a), None)) == B.LS_ERR_UNSUPPORTED
    a.heads = 64
    a.key_scale = None
    assert _err(lib, lib.ls_index_score(C.byref(a), None)) == B.LS_ERR_INVALID_ARG
    a.key_scale = 16
    a.page_table = None
    assert _err(lib, lib.ls_index_score(C.byref(a), None)) == B.LS_ERR_INVALID_ARG
    # misaligned key pool
    a.page_table = 16
    a.key_pool = 17
    assert _err(lib, lib.ls_index_score(C.byref(a), None)) == B.LS_ERR_INVALID_ARG
    # hot buffer: k larger than the buffer, too many slots
    h = B.HotbufArgs(batch=1, k=4097, n_slots=4096, max_len=100, sel=16, sel_score=16, pos_of_slot=16,
                     recent_score=16, slot_of_pos=16, sel_slot=16, miss_pos=16, miss_slot=16, n_miss=16)
    assert _err(lib, lib.ls_hotbuf_resolve(C.byref(h), None)) == B.LS_ERR_INVALID_ARG
    h.k, h.n_slots = 8, 8192
    assert _err(lib, lib.ls_hotbuf_resolve(C.byref(h), None)) == B.LS_ERR_INVALID_ARG
    # gather: row size not a multiple of 16
    g = B.GatherArgs(batch=1, k=8, n_slots=8, max_pages=1, row_bytes=1000, num_pages=1, host_kv=16,
                     page_table=16, miss_pos=16, miss_slot=16, n_miss=16, hbuf=16)
    assert _err(lib, lib.ls_gather_misses(C.byref(g), None)) == B.LS_ERR_INVALID_ARG
    # attention: unsupported MLA shape on the tensor-core path, workspace too small
    s = B.SparseAttnArgs(batch=1, heads=64, dk=576, dv=512, k=2048, dtype=B.LS_BF16, softmax_scale=0.04,
                         addressing=B.LS_ROWS_SLOTS, n_slots=4096, row_stride=576, num_rows=4096, q=16,
                         k_rows=16, v_rows=16, sel=16, o=16, lse=16)
    assert _err(lib, lib.ls_sparse_attn_decode(C.byref(s), None, 0, None)) == B.LS_ERR_UNSUPPORTED
    s.heads = 128
    s.batch = 8
    assert lib.ls_sparse_attn_workspace_size(C.byref(s)) > 0
    assert _err(lib, lib.ls_sparse_attn_decode(C.byref(s), None, 0, None)) == B.LS_ERR_INVALID_ARG


def test_arg_structs_keep_their_tensors_alive():
    """A builder given temporaries (x.to(device) inside the call) must hold them until
    the struct goes away; otherwise their memory is reused before the kernel reads it."""
    import gc
    import weakref

    import torch

    made = []

    def tmp(*shape, dtype=torch.float32):
        t = torch.zeros(*shape, dtype=dtype)
        made.append(weakref.ref(t))
        return t

    a = B.attn_args(q=tmp(2, 128, 576, dtype=torch.bfloat16), k_rows=tmp(4, 64, 576, dtype=torch.bfloat16),
                    sel=tmp(2, 64, dtype=torch.int32), o=tmp(2, 128, 512, dtype=torch.bfloat16), lse=tmp(2, 128),
                    scale=0.1, page_table=tmp(2, 4, dtype=torch.int32))
    ia = B.index_args(q=tmp(2, 64, 128), w=tmp(2, 64), key_pool=tmp(3, 64, 128),
                      page_table=tmp(2, 4, dtype=torch.int32), lens=tmp(2, dtype=torch.int32), scores=tmp(2, 256))
    c = B.c2f_args(index=ia, k=64, summaries=tmp(2, 4, 256, dtype=torch.uint8), block_scale=tmp(2, 4),
                   idx=tmp(2, 64, dtype=torch.int32))
    d = B.decode_step_args(index=ia, k=64, attn=a, idx=tmp(2, 64, dtype=torch.int32))
    del ia, a
    gc.collect()
    assert all(r() is not None for r in made)
    del c, d
    gc.collect()
    assert all(r() is None for r in made)
