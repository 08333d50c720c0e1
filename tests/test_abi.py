"""The C-ABI library loads, exports every declared symbol and validates arguments (CPU only).

No compute call is made here: the checks below all fail host-side validation before any
CUDA call, or are pure host functions.
"""
import ctypes
import os
import re

import pytest

import long_context_sparse_11_b200 as dsa
from long_context_sparse_11_b200 import binding as B
import oracle.dsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\([^;{]*\)\s*;", src)
    return sorted(set(n for n in names if n.startswith(("dsa_", "indexshare_"))))


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_11_b200.build import build
    build()
    return dsa.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)


def test_struct_layouts_match(lib):
    assert lib.dsa_abi_version() == 1
    assert lib.dsa_abi_sizeof(0) == ctypes.sizeof(B.CacheView)
    assert lib.dsa_abi_sizeof(1) == ctypes.sizeof(B.IndexHandle)
    assert lib.dsa_abi_sizeof(2) == ctypes.sizeof(B.GroupArgs)


def test_schedule_agrees_with_oracle(lib):
    for l, full, prod in O.layer_schedule(78):
        assert bool(lib.dsa_layer_is_full(l)) == full
        assert lib.dsa_layer_producer(l) == prod


def test_status_strings(lib):
    for s in range(9):
        assert lib.dsa_status_str(s).decode() != "unknown status"


def _err(lib):
    return lib.dsa_last_error().decode()


def test_host_validation_rejects_before_launch(lib):
    # vec_len other than 128
    assert lib.dsa_quant_e4m3(16, 4, 64, 16, 16, None) == B.DSA_ERR_UNSUPPORTED
    # misaligned pointers
    assert lib.dsa_quant_e4m3(17, 4, 128, 16, 16, None) == B.DSA_ERR_INVALID_ARG
    assert "aligned" in _err(lib)
    # k out of range
    assert lib.dsa_topk(16, 64, 4, None, 1, 64, 0, 16, None, 0, None) == B.DSA_ERR_INVALID_ARG
    assert lib.dsa_topk(16, 64, 4, None, 1, 64, 4096, 16, None, 0, None) == B.DSA_ERR_INVALID_ARG
    # ld not a multiple of 4
    assert lib.dsa_topk(16, 63, 4, None, 1, 63, 8, 16, None, 0, None) == B.DSA_ERR_INVALID_ARG
    # wrong cache dims / dtypes
    v = B.CacheView(16, None, None, None, 128, 100, 64, B.DSA_BF16, 0, 0)
    assert lib.dsa_indexer_score(16, 0, None, 16, 4, 0, ctypes.byref(v), 16, 128, None) == B.DSA_ERR_UNSUPPORTED
    v = B.CacheView(16, None, None, None, 128, 100, 128, B.DSA_BF16, 0, 0)
    assert lib.dsa_indexer_score(16, B.DSA_E4M3, None, 16, 4, 0, ctypes.byref(v), 16, 128, None) \
        == B.DSA_ERR_UNSUPPORTED
    # paged caches must be e4m3 and carry seq_lens
    v = B.CacheView(16, None, 32, None, 576, 6400, 576, B.DSA_BF16, 4, 2)
    assert lib.dsa_sparse_mla_attn(16, ctypes.byref(v), 16, 2, 1, 8, 0.04, 16, None, None, 0, None) \
        == B.DSA_ERR_UNSUPPORTED
    v = B.CacheView(16, 48, 32, None, 576, 6400, 576, B.DSA_E4M3, 4, 2)
    assert lib.dsa_sparse_mla_attn(16, ctypes.byref(v), 16, 2, 1, 8, 0.04, 16, None, None, 0, None) \
        == B.DSA_ERR_INVALID_ARG
    # n_q not a multiple of the rows per index row
    v = B.CacheView(16, None, None, None, 576, 100, 576, B.DSA_BF16, 0, 0)
    assert lib.dsa_sparse_mla_attn(16, ctypes.byref(v), 16, 5, 2, 8, 0.04, 16, None, None, 0, None) \
        == B.DSA_ERR_INVALID_ARG


def test_cache_write_validation(lib):
    args = dict(seq=None, pos=32, bt=48, batch=2, max_pages=4, n_pages=8, pool=64, scale=80)

    def call(x=16, n=4, dim=128, **kw):
        a = dict(args, **kw)
        return lib.dsa_cache_write_e4m3(x, n, dim, a["seq"], a["pos"], a["bt"], a["batch"], a["max_pages"],
                                        a["n_pages"], a["pool"], a["scale"], None)
    assert call(dim=512) == B.DSA_ERR_UNSUPPORTED           # neither an index key nor a latent row
    assert call(n=-1) == B.DSA_ERR_INVALID_ARG
    assert call(x=17) == B.DSA_ERR_INVALID_ARG and "aligned" in _err(lib)
    assert call(pool=65) == B.DSA_ERR_INVALID_ARG
    assert call(pos=None) == B.DSA_ERR_INVALID_ARG
    assert call(n_pages=0) == B.DSA_ERR_INVALID_ARG and "empty" in _err(lib)
    assert call(n=0) == B.DSA_OK                            # nothing to write: no launch


def test_per_row_paged_view_repeats_tables_not_pages():
    import torch
    pool = torch.zeros(6, 64, 128, dtype=torch.uint8)
    scale = torch.ones(6, 64)
    bt = torch.tensor([[4, 1, -1], [0, 5, 2]], dtype=torch.int32)
    lens = torch.tensor([100, 150], dtype=torch.int32)
    v = dsa.paged_view(pool, scale, bt, lens, rows_per_seq=3)
    assert v.batch == 6 and v.max_pages == 3 and v.data == pool.data_ptr() and v.n_tokens == 6 * 64
    assert v._keep[2].tolist() == [[4, 1, -1]] * 3 + [[0, 5, 2]] * 3
    assert v._keep[3].tolist() == [100] * 3 + [150] * 3
    assert v.block_table == v._keep[2].data_ptr() and v.seq_lens == v._keep[3].data_ptr()


def test_empty_inputs_are_a_no_op(lib):
    """Zero rows (an empty batch, a chunk with no queries) succeed with no launch and no device
    access, whatever the data pointers are."""
    before = lib.dsa_launch_count()
    assert lib.dsa_quant_e4m3(None, 0, 128, None, None, None) == B.DSA_OK
    v = B.CacheView(16, None, None, None, 128, 100, 128, B.DSA_BF16, 0, 0)
    assert lib.dsa_indexer_score(None, B.DSA_BF16, None, None, 0, 0, ctypes.byref(v), None, 128, None) == B.DSA_OK
    assert lib.dsa_topk(None, 64, 0, None, 1, 64, 8, None, None, 0, None) == B.DSA_OK
    assert lib.dsa_topk_no_alloc(None, 64, 0, None, 1, 64, 8, None, None) == B.DSA_OK
    v = B.CacheView(16, None, None, None, 576, 100, 576, B.DSA_BF16, 0, 0)
    assert lib.dsa_sparse_mla_attn(None, ctypes.byref(v), None, 0, 1, 8, 0.04, None, None, None, 0, None) == B.DSA_OK
    assert lib.dsa_cache_write_e4m3(None, 0, 576, None, None, None, 1, 1, 1, None, None, None) == B.DSA_OK
    assert lib.dsa_launch_count() == before


def test_group_handle_checks(lib):
    a = B.GroupArgs()
    a.q_idx, a.w = 16, 32
    a.idx_keys = B.CacheView(16, None, None, None, 128, 100, 128, B.DSA_BF16, 0, 0)
    a.indexer_dtype, a.n_idx_rows, a.k, a.q_rows_per_idx_row, a.n_layers = B.DSA_BF16, 100, 64, 1, 2
    a.softmax_scale = 0.04
    for i in range(2):
        a.q[i], a.out[i] = 64, 128
        a.kv[i] = B.CacheView(16, None, None, None, 576, 100, 576, B.DSA_BF16, 0, 0)
    # handle of the wrong size for a reuse call: stale
    h = B.IndexHandle(256, 100, 32, 1, 0, 1)
    assert lib.indexshare_group_forward(ctypes.byref(a), ctypes.byref(h), 1, None) == B.DSA_ERR_STALE_HANDLE
    # unfilled handle for a reuse call: stale
    h = B.IndexHandle(256, 100, 64, 0, -1, 0)
    assert lib.indexshare_group_forward(ctypes.byref(a), ctypes.byref(h), 1, None) == B.DSA_ERR_STALE_HANDLE
    assert "unfilled" in _err(lib)
    # a fill that fails leaves the handle unfilled, so a reuse call cannot accept indices that the
    # failed fill may have half overwritten.  No workspace is given: the fill fails before any
    # launch, for want of a device here or of the workspace on a GPU machine.
    assert a.workspace is None and a.workspace_bytes == 0
    h = B.IndexHandle(256, 100, 64, 1, 0, 3)
    rc = lib.indexshare_group_forward(ctypes.byref(a), ctypes.byref(h), 0, None)
    assert rc in (B.DSA_ERR_CUDA, B.DSA_ERR_WORKSPACE)
    assert h.filled == 0 and h.generation == 3
    assert lib.indexshare_group_forward(ctypes.byref(a), ctypes.byref(h), 1, None) == B.DSA_ERR_STALE_HANDLE
    # too many layers
    a.n_layers = 5
    assert lib.indexshare_group_forward(ctypes.byref(a), ctypes.byref(h), 0, None) == B.DSA_ERR_INVALID_ARG


def test_product_path_never_imports_oracle():
    pkg = os.path.join(ROOT, "long_context_sparse_11_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f


def test_projection_arguments_are_checked(lib):
    # widths that are not multiples of 64, and a missing workspace, fail before any launch
    assert lib.dsa_indexer_project(16, 16, 16, 16, 16, 16, 4, 100, 6144, 16, 16, 16, 16, 1 << 20, None) == \
        B.DSA_ERR_UNSUPPORTED
    assert lib.dsa_indexer_project(16, 16, 16, 16, 16, 16, 4, 2048, 6144, 16, 16, 16, 16, 8, None) == \
        B.DSA_ERR_WORKSPACE
    assert lib.dsa_mla_latent(16, 16, 16, 16, 4, 6144, 0.5, 16, 16, 1 << 20, None) == B.DSA_ERR_INVALID_ARG


def test_every_kernel_launched_with_programmatic_dependency_waits_first():
    """Kernels launched with programmatic stream serialisation may start before the previous
    kernel of the stream has finished; each must wait for it (grid_dependency_sync) before its
    first memory access, or stream order no longer holds.  Checked on the sources: every kernel
    named in a launch_pdl call opens with that wait."""
    csrc = os.path.join(ROOT, "long_context_sparse_11_b200", "csrc")
    lib_src = open(os.path.join(csrc, "dsa_lib.cu")).read()
    launched = set(re.findall(r"launch_pdl\(\s*(?:\w+::)*(\w+)\s*[<,]", lib_src))
    assert {"sparse_mla_kernel", "combine_kernel", "indexer_kernel", "topk_seg_filter_kernel"} <= launched
    bodies = {}
    for f in os.listdir(csrc):
        src = open(os.path.join(csrc, f)).read()
        for m in re.finditer(r"__global__\s+void\s+(?:__launch_bounds__\([^)]*\)\s*)?(\w+)\s*\(", src):
            brace = src.index("{", m.end())
            bodies[m.group(1)] = src[brace + 1:brace + 200]
    for name in sorted(launched):
        assert name in bodies, name
        first = bodies[name].strip().split(";")[0].strip()
        assert first == "grid_dependency_sync()", (name, first)
