"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every entry point include/seer.h declares, and
reject bad arguments on the host with the documented status before touching
the device.
"""
import ctypes
import subprocess

import pytest

from block_sparse_attention_seer_b200 import api


def test_header_declares_the_path_calls():
    names = api.header_functions()
    for n in ("seer_kpool_update", "seer_gate_scores", "seer_select_blocks", "seer_sparse_decode",
              "seer_combine", "seer_status_string", "seer_default_num_splits"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", api._build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in api.header_functions():
        assert n in exported, n
        assert hasattr(api.LIB, n)


def test_status_strings():
    assert api.status_string(0) == "ok"
    assert api.status_string(1) == "invalid argument"
    assert api.status_string(2) == "unsupported size"
    assert api.status_string(3) == "CUDA error"


def _dims(**kw):
    d = dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, gate_dim=128, block_size=64, max_seq_len=1024)
    d.update(kw)
    return api.make_dims(**d)


FAKE = 1 << 20  # never dereferenced: validation fails before any launch


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), api.SEER_ERR_UNSUPPORTED),
    (dict(gate_dim=32), api.SEER_ERR_UNSUPPORTED),
    (dict(block_size=32), api.SEER_ERR_UNSUPPORTED),
    (dict(num_q_heads=18, num_kv_heads=2), api.SEER_ERR_UNSUPPORTED),   # G = 9
    (dict(num_q_heads=7), api.SEER_ERR_INVALID_ARG),                     # not a multiple of Hkv
    (dict(batch=0), api.SEER_ERR_INVALID_ARG),
    (dict(max_seq_len=0), api.SEER_ERR_INVALID_ARG),
    (dict(max_seq_len=(1 << 24) + 1), api.SEER_ERR_UNSUPPORTED),
])
def test_bad_dims_rejected(bad, status):
    d = _dims(**bad)
    st = api.LIB.seer_combine(ctypes.byref(d), FAKE, FAKE, 4, FAKE, None, None)
    assert st == status
    st = api.LIB.seer_sparse_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 4, 0.0, FAKE, FAKE, None)
    assert st == status


def test_null_pointers_and_bad_scalars_rejected():
    d = _dims()
    L = api.LIB
    assert L.seer_kpool_update(None, FAKE, FAKE, FAKE, None, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_kpool_update(ctypes.byref(d), None, FAKE, FAKE, None, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_gate_scores(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks(ctypes.byref(d), FAKE, FAKE, 0, FAKE, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks(ctypes.byref(d), FAKE, FAKE, 64, None, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_sparse_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 0.0, FAKE, FAKE,
                                None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_sparse_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 0, 0.0, FAKE, FAKE,
                                None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_sparse_decode(ctypes.byref(d), FAKE + 2, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 4, 0.0, FAKE, FAKE,
                                None) == api.SEER_ERR_INVALID_ARG            # q not 16-byte aligned
    assert L.seer_sparse_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 4, float("nan"), FAKE,
                                FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_combine(ctypes.byref(d), FAKE, FAKE, 0, FAKE, None, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_combine(ctypes.byref(d), None, FAKE, 4, FAKE, None, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_default_num_splits(0, ctypes.byref(ctypes.c_int32())) == api.SEER_ERR_INVALID_ARG


def test_gate_variants_validate_on_host():
    d = _dims()
    L = api.LIB
    assert L.seer_gate_scores_agg(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 3, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_gate_scores_agg(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, -1, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_gate_scores_agg(ctypes.byref(d), None, FAKE, FAKE, FAKE, 0, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks_threshold(ctypes.byref(d), FAKE, FAKE, 64, float("nan"), FAKE, FAKE,
                                          None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks_threshold(ctypes.byref(d), FAKE, FAKE, 100, 0.0, FAKE, FAKE,
                                          None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_select_blocks_threshold(ctypes.byref(d), FAKE, FAKE, 64, 0.0, None, FAKE,
                                          None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_block_mass(ctypes.byref(d), FAKE, FAKE, FAKE, float("inf"), FAKE, None,
                             None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_block_mass(ctypes.byref(d), FAKE, FAKE, FAKE, 0.0, None, None, None) == api.SEER_ERR_INVALID_ARG


def test_append_kv_validates_on_host():
    d = _dims()
    L = api.LIB
    assert L.seer_append_kv(None, FAKE, FAKE, FAKE, FAKE, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_append_kv(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_append_kv(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_append_kv(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE + 8, FAKE, None) == api.SEER_ERR_INVALID_ARG
    bad = _dims(head_dim=96)
    assert L.seer_append_kv(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, None) == api.SEER_ERR_UNSUPPORTED


def test_prefill_validates_on_host():
    d = _dims()
    L = api.LIB
    bad, unsup = api.SEER_ERR_INVALID_ARG, api.SEER_ERR_UNSUPPORTED
    assert L.seer_prefill_gate_scores(None, FAKE, FAKE, FAKE, FAKE, FAKE, None) == bad
    assert L.seer_prefill_gate_scores(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, None) == bad
    assert L.seer_prefill_select_blocks(ctypes.byref(d), FAKE, FAKE, 100, FAKE, FAKE, None) == bad  # not k * blk
    assert L.seer_prefill_select_blocks(ctypes.byref(d), FAKE, FAKE, 0, FAKE, FAKE, None) == bad
    attn = L.seer_prefill_attention
    assert attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0.0, FAKE, None, None) == bad  # kmax < 1
    assert attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, None, None, None) == bad  # no out
    assert attn(ctypes.byref(d), FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, FAKE, None, None) == bad  # q
    assert attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, FAKE + 8, None, None) == bad  # out
    assert attn(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, float("nan"), FAKE, None, None) == bad
    many_blocks = _dims(max_seq_len=4097 * 64)  # more than 4096 query blocks
    assert attn(ctypes.byref(many_blocks), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, FAKE, None, None) == unsup
    # 4096 blocks, but 128 x 64 query rows of 262144 tokens do not fit a 32-bit TMA row coordinate
    wide = _dims(batch=128, num_q_heads=64, num_kv_heads=8, max_seq_len=4096 * 64)
    assert attn(ctypes.byref(wide), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0.0, FAKE, None, None) == unsup


def test_python_wrapper_raises_on_error():
    with pytest.raises(api.SeerError) as e:
        api.seer_combine(_dims(head_dim=96), FAKE, FAKE, 4, FAKE, None, stream=0)
    assert e.value.status == api.SEER_ERR_UNSUPPORTED


def test_failure_detection_entries_validate_on_host():
    L = api.LIB
    assert L.seer_decode_wait_failures(None, 0) == api.SEER_ERR_INVALID_ARG
    assert L.seer_wait_selftest(-1, ctypes.byref(ctypes.c_int32())) == api.SEER_ERR_INVALID_ARG
    assert L.seer_wait_selftest(3_000_000_000, ctypes.byref(ctypes.c_int32())) == api.SEER_ERR_INVALID_ARG
    assert L.seer_wait_selftest(1000, None) == api.SEER_ERR_INVALID_ARG


def test_decode_step_validates_on_host():
    d = _dims()
    L = api.LIB
    args = [FAKE] * 6
    sz = ctypes.c_size_t(0)
    assert L.seer_decode_step_workspace_size(ctypes.byref(d), 100, ctypes.byref(sz)) == api.SEER_ERR_INVALID_ARG
    assert L.seer_decode_step_workspace_size(ctypes.byref(d), 64, None) == api.SEER_ERR_INVALID_ARG
    assert L.seer_decode_step(ctypes.byref(_dims(head_dim=96)), *args, None, 64, 0.0, FAKE, FAKE, FAKE, FAKE, None,
                              FAKE, 1 << 30, None) == api.SEER_ERR_UNSUPPORTED
    assert L.seer_decode_step(ctypes.byref(d), *args, None, 64, 0.0, FAKE, FAKE, FAKE, FAKE, None, None, 1 << 30,
                              None) == api.SEER_ERR_INVALID_ARG           # no workspace
    assert L.seer_decode_step(ctypes.byref(d), *args, None, 100, 0.0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30,
                              None) == api.SEER_ERR_INVALID_ARG           # budget not a multiple of blk
    assert L.seer_decode_step(ctypes.byref(d), *args, None, 64, 0.0, FAKE, FAKE, FAKE, FAKE, None, FAKE + 16,
                              1 << 30, None) == api.SEER_ERR_INVALID_ARG  # workspace not 256-byte aligned
