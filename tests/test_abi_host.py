"""Host side of the C ABI (no GPU needed): the library loads, exports every symbol that
include/vx.h declares, and rejects bad arguments with the documented status before
launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_block_sparse_kv_b200 import vx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vx.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vx_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(vx.LIB_PATH):
        pytest.skip("libvx.so not built")
    return vx.lib()


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(vx.EXPORTS)


def test_noalloc_scratch_size_matches_the_header():
    m = re.search(r"#define VX_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", open(HEADER).read())
    assert m and int(m.group(1)) << int(m.group(2)) == vx.NOALLOC_SCRATCH_BYTES


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", vx.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in _declared():
        assert name in exported, name
        assert hasattr(L, name)


def test_no_oracle_in_the_product(L):
    # the product library links nothing from the oracle
    out = subprocess.run(["nm", "-D", vx.LIB_PATH], capture_output=True, text=True, check=True).stdout
    assert "orc_" not in out


def _geo(**kw):
    g = dict(batch=2, num_q_heads=16, num_kv_heads=8, head_dim_qk=128, head_dim_v=128, page_size=16,
             mla_shared_kv=0, num_pool_pages=100)
    g.update(kw)
    return vx.vx_geometry(**g)


def _table(max_pages=10, ptr=256):
    return vx.vx_page_table(ptr, ptr, ptr, max_pages)


FAKE = 4096  # an aligned non-NULL address; validation fails before anything dereferences it


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), vx.VX_ERR_INVALID_ARG),
    (dict(num_q_heads=12, num_kv_heads=8), vx.VX_ERR_INVALID_ARG),
    (dict(num_pool_pages=0), vx.VX_ERR_INVALID_ARG),
    (dict(page_size=8), vx.VX_ERR_UNSUPPORTED),
    (dict(head_dim_qk=96, head_dim_v=96), vx.VX_ERR_UNSUPPORTED),
    (dict(head_dim_v=64), vx.VX_ERR_UNSUPPORTED),
    (dict(num_q_heads=8 * 32), vx.VX_ERR_UNSUPPORTED),
    (dict(num_q_heads=12, num_kv_heads=3), vx.VX_ERR_UNSUPPORTED),
    (dict(num_q_heads=32, num_kv_heads=32), vx.VX_ERR_UNSUPPORTED),
    (dict(mla_shared_kv=1), vx.VX_ERR_UNSUPPORTED),
    (dict(mla_shared_kv=1, num_kv_heads=1, num_q_heads=32, head_dim_qk=576, head_dim_v=512, page_size=64),
     vx.VX_ERR_UNSUPPORTED),
])
def test_bad_geometry_is_rejected_before_launch(L, kw, status):
    g = _geo(**kw)
    t = _table()
    st = L.vx_score_pages(ctypes.byref(g), ctypes.byref(t), FAKE, FAKE, 0, FAKE, None, None)
    assert st == status, L.vx_last_error()
    assert L.vx_last_error().decode()
    assert L.vx_workspace_size(ctypes.byref(g), 10, 4, 8) == 0


def test_bad_pointers_and_sizes(L):
    g, t = _geo(), _table()
    gp, tp = ctypes.byref(g), ctypes.byref(t)
    assert L.vx_score_pages(None, tp, FAKE, FAKE, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_score_pages(gp, None, FAKE, FAKE, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_score_pages(gp, tp, None, FAKE, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_score_pages(gp, tp, FAKE + 2, FAKE, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG  # misaligned
    assert L.vx_score_pages(gp, tp, FAKE, FAKE, 12, FAKE, None, None) == vx.VX_ERR_INVALID_ARG  # not /8
    assert L.vx_score_pages(gp, tp, FAKE, FAKE, 136, FAKE, None, None) == vx.VX_ERR_INVALID_ARG  # > dqk
    bad_table = _table(max_pages=0)
    assert L.vx_score_pages(gp, ctypes.byref(bad_table), FAKE, FAKE, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_topk_pages(gp, tp, FAKE, 0, 0, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG  # k = 0
    assert L.vx_topk_pages(gp, tp, FAKE, 4, 4, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG  # mode 4
    assert L.vx_centroid_update(gp, tp, None, None, FAKE, None, None, None, None, None) == vx.VX_ERR_INVALID_ARG
    # append needs v_new for GQA
    assert L.vx_centroid_update(gp, tp, FAKE, FAKE, FAKE, FAKE, None, None, None, None) == vx.VX_ERR_INVALID_ARG
    # prefill write (k_new and first_pos): GQA needs v_cache and v_new; first_pos must be 4-byte aligned
    assert L.vx_centroid_update(gp, tp, FAKE, None, FAKE, FAKE, FAKE, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_centroid_update(gp, tp, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_centroid_update(gp, tp, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, None, None) == vx.VX_ERR_INVALID_ARG
    assert L.vx_centroid_update(gp, tp, FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    # decode: workspace checked before launch (explicit split count: no device query needed)
    assert L.vx_sparse_decode(gp, tp, FAKE, FAKE, FAKE, FAKE, 4, ctypes.c_float(0.0), 8, FAKE, None, None, 0,
                              None, None) == vx.VX_ERR_WORKSPACE
    need = L.vx_workspace_size(gp, 10, 4, 8)
    assert need > 0
    # the decode call needs only its split partials: (rows + splits) * G * (Dv + 2) floats, 256-aligned
    rows, G = 2 * 8, 2
    partial = -(-(rows + 8) * G * 128 * 4 // 256) * 256 + -(-(rows + 8) * G * 2 * 4 // 256) * 256
    assert partial < need
    assert L.vx_sparse_decode(gp, tp, FAKE, FAKE, FAKE, FAKE, 4, ctypes.c_float(0.0), 8, FAKE, None, FAKE,
                              partial - 1, None, None) == vx.VX_ERR_WORKSPACE
    assert b"needed" in L.vx_last_error()
    assert L.vx_sparse_decode(gp, tp, FAKE, FAKE, FAKE, FAKE, 4, ctypes.c_float(float("nan")), 8, FAKE, None,
                              FAKE, need, None, None) == vx.VX_ERR_INVALID_ARG


def test_appending_step_validation(L):
    # vx_block_topk_decode_append needs k_new (and v_new for GQA) and checks the step's arguments
    # before any launch (explicit split count: no device query needed)
    gp, tp = ctypes.byref(_geo()), ctypes.byref(_table())
    f0 = ctypes.c_float(0.0)
    args = lambda k_new, v_new, ws_bytes: (gp, tp, FAKE, FAKE, FAKE, FAKE, k_new, v_new, 4, 0, 0, f0, 0, 8, FAKE,
                                           None, None, None, FAKE, ws_bytes, None, None)
    assert L.vx_block_topk_decode_append(*args(None, FAKE, 1 << 30)) == vx.VX_ERR_INVALID_ARG
    assert b"k_new" in L.vx_last_error()
    assert L.vx_block_topk_decode_append(*args(FAKE, None, 1 << 30)) == vx.VX_ERR_INVALID_ARG
    assert L.vx_block_topk_decode_append(*args(FAKE + 8, FAKE, 1 << 30)) == vx.VX_ERR_INVALID_ARG  # misaligned
    assert L.vx_block_topk_decode_append(*args(FAKE, FAKE, 16)) == vx.VX_ERR_WORKSPACE


def test_table_ready_flag_validation(L):
    # VX_TABLE_READY is a flag of the chained steps' mode only; other bits are rejected
    gp, tp = ctypes.byref(_geo()), ctypes.byref(_table())
    f0 = ctypes.c_float(0.0)
    step = lambda mode, ws_bytes: L.vx_block_topk_decode(gp, tp, FAKE, FAKE, FAKE, FAKE, 4, mode, 0, f0, 0, 8, FAKE,
                                                         None, None, None, FAKE, ws_bytes, None, None)
    assert step(vx.VX_TABLE_READY | 1, 16) == vx.VX_ERR_WORKSPACE  # the mode passed, the workspace did not
    assert step(vx.VX_TABLE_READY << 1, 1 << 30) == vx.VX_ERR_INVALID_ARG
    assert step(vx.VX_TABLE_READY | 4, 1 << 30) == vx.VX_ERR_INVALID_ARG
    assert L.vx_topk_pages(gp, tp, FAKE, 4, vx.VX_TABLE_READY, 0, FAKE, None, None) == vx.VX_ERR_INVALID_ARG
    hdr = open(os.path.join(ROOT, "include", "vx.h")).read()
    assert f"#define VX_TABLE_READY {vx.VX_TABLE_READY:#x}" in hdr


def test_persistent_step_validation(L):
    # vx_block_topk_decode_persistent refuses what it cannot run, before any launch
    tp = ctypes.byref(_table())
    f0 = ctypes.c_float(0.0)
    mla = _geo(num_q_heads=16, num_kv_heads=1, head_dim_qk=576, head_dim_v=512, page_size=64, mla_shared_kv=1)
    assert L.vx_block_topk_decode_persistent(ctypes.byref(mla), tp, FAKE, FAKE, FAKE, FAKE, 4, f0, FAKE, None, None,
                                             None, FAKE, 1 << 30, None, None) == vx.VX_ERR_UNSUPPORTED
    gp = ctypes.byref(_geo())
    assert L.vx_block_topk_decode_persistent(gp, tp, None, FAKE, FAKE, FAKE, 4, f0, FAKE, None, None, None, FAKE,
                                             1 << 30, None, None) == vx.VX_ERR_INVALID_ARG  # q NULL
    assert L.vx_block_topk_decode_persistent(gp, tp, FAKE, FAKE, FAKE, FAKE, 0, f0, FAKE, None, None, None, FAKE,
                                             1 << 30, None, None) == vx.VX_ERR_INVALID_ARG  # k = 0
    assert L.vx_block_topk_decode_persistent(gp, tp, FAKE, FAKE, None, FAKE, 4, f0, FAKE, None, None, None, FAKE,
                                             1 << 30, None, None) == vx.VX_ERR_INVALID_ARG  # v_cache NULL


def test_workspace_size_is_deterministic_and_monotone(L):
    g = _geo()
    gp = ctypes.byref(g)
    a = L.vx_workspace_size(gp, 100, 16, 64)
    assert a == L.vx_workspace_size(gp, 100, 16, 64)
    assert L.vx_workspace_size(gp, 200, 16, 64) > a  # more pages -> larger score rows
    assert L.vx_workspace_size(gp, 100, 32, 64) > a  # larger k
    assert L.vx_workspace_size(gp, 100, 16, 128) > a  # more splits -> more partials
    assert a % 256 == 0


def test_status_strings(L):
    assert L.vx_status_string(0) == b"VX_OK"
    assert L.vx_status_string(3) == b"VX_ERR_WORKSPACE"
    assert b"sm_100a" in L.vx_version()
