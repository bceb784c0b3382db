"""CPU-only checks of the C-ABI library: it builds for sm_100a, loads, exports
every symbol the header declares, and rejects invalid arguments on the host
before touching any device."""
import ctypes
import os
import re

import pytest

import flash_attention_fwd_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "varlen_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(varlen_attn_[a-z_0-9]+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_exported_symbols():
    assert header_functions() == sorted(fa.EXPORTED_SYMBOLS)


def test_library_loads_and_exports_every_symbol():
    lib = fa.load_library()
    raw = ctypes.CDLL(fa.LIB_PATH)
    for name in header_functions():
        assert hasattr(raw, name), name
    assert lib.varlen_attn_abi_version() == 6


def test_library_is_built_for_sm100a():
    data = open(fa.LIB_PATH, "rb").read()
    # the fatbin names its target architecture; only sm_100a is built
    assert b"sm_100a" in data


def test_strerror_covers_codes():
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, -99):
        msg = fa.strerror(code)
        assert isinstance(msg, str) and msg


BASE = dict(q_ptr=0x10000, k_ptr=0x20000, v_ptr=0x30000, cu_q_ptr=0x40000, cu_k_ptr=0x50000,
            batch=2, total_q=10, total_k=10, max_seqlen_q=5, max_seqlen_k=5, num_heads=4,
            num_kv_heads=2, head_dim=128, causal=True, scale=0.0, dtype_code=0,
            out_ptr=0x60000, lse_ptr=0x70000, stream=0)


# paged K/V: 4 pages of 16 keys, cu_seqlens_k unused
PAGED = dict(page_table_ptr=0x90000, page_table_stride=2, page_size=16, total_k=64,
             seqused_k_ptr=0x80000, cu_k_ptr=0)


@pytest.mark.parametrize("change,code", [
    (dict(num_heads=5), -2),                 # H % Hkv != 0
    (dict(head_dim=96), -2),                 # unsupported D
    (dict(head_dim=32), -2),
    (dict(batch=-1), -2),
    (dict(total_q=-3), -2),
    (dict(total_q=1 << 31), -2),
    (dict(max_seqlen_k=-1), -2),
    (dict(num_kv_heads=0), -2),
    (dict(dtype_code=2), -3),
    (dict(q_ptr=0), -1),
    (dict(out_ptr=0), -1),
    (dict(lse_ptr=0), -1),
    (dict(k_ptr=0), -1),
    (dict(cu_q_ptr=0), -1),
    (dict(q_ptr=0x10008), -4),               # 8-byte aligned only
    (dict(out_ptr=0x60002), -4),
    (dict(lse_ptr=0x70002), -4),
    (dict(cu_k_ptr=0x50001), -4),
    # the v2 entry point (window / seqused_k) validates the same way
    (dict(window_left=4, num_heads=5), -2),
    (dict(window_right=0, head_dim=96), -2),
    (dict(seqused_k_ptr=0x80000, dtype_code=7), -3),
    (dict(window_left=2, q_ptr=0), -1),
    (dict(seqused_k_ptr=0x80002), -4),       # seqused_k needs 4-byte alignment
    (dict(window_left=1, window_right=1, lse_ptr=0x70001), -4),
    # the v3 entry point (paged K/V)
    (dict(PAGED, page_size=24), -2),         # not a multiple of 16
    (dict(PAGED, page_size=0), -2),
    (dict(PAGED, total_k=40), -2),           # not a whole number of pages
    (dict(PAGED, page_table_stride=0), -2),
    (dict(PAGED, seqused_k_ptr=0), -1),      # a page table needs seqused_k
    (dict(PAGED, cu_q_ptr=0), -1),
    (dict(PAGED, page_table_ptr=0x90002), -4),
    (dict(PAGED, num_heads=5), -2),
    (dict(sinks_ptr=0x90002), -4),           # sinks need 4-byte alignment
    (dict(sinks_ptr=0x90000, head_dim=48), -2),
    # the v4 entry point (key-range split): the piece count must be in [0, 32]
    (dict(num_splits=33, causal=False), -2),
    (dict(num_splits=-2, causal=False), -2),
    (dict(num_splits=4, num_heads=5), -2),
    (dict(num_splits=0, q_ptr=0x10004), -4),
])
def test_host_validation_rejects(change, code):
    args = dict(BASE)
    args.update(change)
    assert fa.varlen_attn_fwd_raw(**args) == code


def test_empty_problems_are_noops_without_device():
    args = dict(BASE)
    args.update(batch=0)
    assert fa.varlen_attn_fwd_raw(**args) == 0
    args = dict(BASE)
    args.update(total_q=0, q_ptr=0, out_ptr=0, lse_ptr=0)
    assert fa.varlen_attn_fwd_raw(**args) == 0
    args = dict(BASE)
    args.update(batch=0, window_left=8, window_right=0, seqused_k_ptr=0x80000)
    assert fa.varlen_attn_fwd_raw(**args) == 0
    args = dict(BASE)
    args.update(PAGED, total_q=0, q_ptr=0, out_ptr=0, lse_ptr=0)
    assert fa.varlen_attn_fwd_raw(**args) == 0


def test_v4_empty_problem_is_a_noop_without_workspace():
    args = dict(BASE)
    args.update(batch=0, num_splits=8, causal=False)
    assert fa.varlen_attn_fwd_raw(**args) == 0


def test_split_heuristic_and_workspace_size():
    # the short-query / long-KV batch (32 sequences, 1267 queries, 145,046
    # keys, H=32, Hkv=4, D=128) has about 200 work items: no split on 148 SMs
    shortq = (32, 1267, 145046, 64, 7954, 32, 4, 128)
    assert fa.fwd_num_splits(*shortq, num_sms=148) == 1
    # ... but with many more SMs than items, pieces fill them
    assert fa.fwd_num_splits(*shortq, num_sms=1000) > 1
    # decode-like: 8 sequences of one query, 8 KV heads (64 items), 32k keys
    dec = (8, 8, 8 * 32768, 1, 32768, 32, 8, 128)
    n = fa.fwd_num_splits(*dec, num_sms=148)
    assert n == 8  # 256 key tiles: 16 pieces of 16, capped at 8 with replicated rows
    # without replicated rows (8 query heads per KV head -> 8 rows, but
    # max_seqlen_q = 5 -> 40 rows > 32): 16
    assert fa.fwd_num_splits(8, 40, 8 * 32768, 5, 32768, 64, 8, 128, num_sms=148) == 16
    # never with a causal rule or a window, never pieces under 16 key tiles
    assert fa.fwd_num_splits(*dec, causal=True, num_sms=148) == 1
    assert fa.fwd_num_splits(*dec, window_size_left=100, num_sms=148) == 1
    assert fa.fwd_num_splits(*dec, window_size_right=0, num_sms=148) == 1
    assert fa.fwd_num_splits(8, 8, 8 * 2048, 1, 2048, 32, 8, 128, num_sms=148) == 1
    assert fa.fwd_num_splits(8, 8, 8 * 4096, 1, 4096, 32, 8, 128, num_sms=148) == 2
    # long prefill: plenty of items, no split
    assert fa.fwd_num_splits(16, 65536, 65536, 24865, 24865, 64, 8, 128, num_sms=148) == 1
    # one sequence, one KV head (8 rows, replicated): at most 8 pieces
    assert fa.fwd_num_splits(1, 1, 1 << 20, 1, 1 << 20, 8, 1, 128, num_sms=148) == 8
    with pytest.raises(fa.VarlenAttnError):
        fa.fwd_num_splits(2, 10, 10, 5, 5, 5, 2, 128, num_sms=148)
    # workspace: pieces x rows x (D + 1) float32; max_seqlen_k = 7954 is 63 key
    # tiles: 4 pieces of up to 16 tiles (H/Hkv = 8, max_seqlen_q = 64: 512
    # rows per item, no replicated rows)
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 7954, 4) == 4 * 1267 * 32 * 129 * 4
    # 63 tiles in at most 5 pieces: 13 tiles a piece, 5 pieces
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 7954, 5) == 5 * 1267 * 32 * 129 * 4
    # 63 tiles in at most 32 pieces: 2 tiles a piece -> 32 pieces (D = 64, no GQA packing)
    assert fa.fwd_workspace_size(10, 4, 4, 64, 5, 7954, 32) == 32 * 10 * 4 * 65 * 4
    # no split and no replicated rows: nothing
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 7954, 1) == 0
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 128, 8) == 0
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 7954, 33) == 0
    assert fa.fwd_workspace_size(1267, 32, 4, 128, 64, 7954, 0) == 0
    # replicated rows (1 query x 4 heads per KV head, keys >= 1024): 4 copies of
    # each key piece, at most 8 key pieces
    assert fa.fwd_workspace_size(8, 32, 8, 128, 1, 4096, 1) == 4 * 8 * 32 * 129 * 4
    assert fa.fwd_workspace_size(8, 32, 8, 128, 1, 4096, 2) == 8 * 8 * 32 * 129 * 4
    assert fa.fwd_workspace_size(8, 32, 8, 128, 1, 32768, 16) == 32 * 8 * 32 * 129 * 4
    # ... not for 8 query tokens x 8 heads (64 rows), nor for short key ranges
    assert fa.fwd_workspace_size(64, 32, 4, 128, 8, 4096, 1) == 0
    assert fa.fwd_workspace_size(8, 32, 8, 128, 1, 1000, 1) == 0
    # the auto piece count with replicated rows: about 32 key tiles a piece, at
    # most 8 pieces, none with plenty of items
    assert fa.fwd_num_splits(8, 8, 8 * 32768, 1, 32768, 32, 8, 128, num_sms=148) == 8
    assert fa.fwd_num_splits(64, 64, 64 * 8000, 1, 16384, 32, 8, 128, num_sms=148) == 4
    assert fa.fwd_num_splits(512, 512, 512 * 8000, 1, 16384, 32, 8, 128, num_sms=148) == 1


def test_product_module_does_not_import_oracle():
    import sys
    pkg_dir = os.path.dirname(fa.__file__)
    for fn in os.listdir(pkg_dir):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg_dir, fn)).read()
            assert "oracle" not in re.sub(r'""".*?"""', "", src, flags=re.S), fn


BWD = dict(dout_ptr=0x11000, q_ptr=0x10000, k_ptr=0x20000, v_ptr=0x30000, out_ptr=0x60000,
           lse_ptr=0x70000, cu_q_ptr=0x40000, cu_k_ptr=0x50000, batch=2, total_q=10,
           total_k=10, max_seqlen_q=5, max_seqlen_k=5, num_heads=4, num_kv_heads=2,
           head_dim=128, causal=True, scale=0.0, dtype_code=0, dq_ptr=0x61000,
           dk_ptr=0x62000, dv_ptr=0x63000, workspace_ptr=0x80000, workspace_bytes=4096,
           stream=0)


@pytest.mark.parametrize("change,code", [
    (dict(head_dim=96), -2),                 # the backward covers D = 64, 128, 256
    (dict(num_heads=5), -2),
    (dict(dtype_code=3), -3),
    (dict(dout_ptr=0), -1),
    (dict(dk_ptr=0), -1),
    (dict(cu_k_ptr=0), -1),
    (dict(dq_ptr=0x61008), -4),
    (dict(workspace_ptr=0x80008), -4),
    (dict(workspace_ptr=0), -8),
    (dict(workspace_bytes=100), -8),         # needs 10 * 4 * 4 bytes rounded up to 256
])
def test_backward_host_validation_rejects(change, code):
    args = dict(BWD)
    args.update(change)
    assert fa.varlen_attn_bwd_raw(**args) == code


def test_backward_workspace_size_and_empty_call():
    assert fa.bwd_workspace_size(10, 4) == 256
    assert fa.bwd_workspace_size(1000, 3) == 12032
    assert fa.bwd_workspace_size(0, 4) == 0
    args = dict(BWD)
    args.update(batch=0)
    assert fa.varlen_attn_bwd_raw(**args) == 0


def test_noalloc_backward_rejects_before_any_device_call():
    lib = fa.load_library()
    V = ctypes.c_void_p
    args = dict(BWD)
    # 2^20 query rows x 8 heads x 4 bytes of scratch = 32 MiB > the fixed 16 MiB
    rc = lib.varlen_attn_bwd_noalloc(*(V(args[n]) for n in (
        "dout_ptr", "q_ptr", "k_ptr", "v_ptr", "out_ptr", "lse_ptr", "cu_q_ptr", "cu_k_ptr")),
        2, 1 << 20, 10, 5, 5, 8, 2, 128, 1, 0.0, 0, V(0x61000), V(0x62000), V(0x63000), V(0))
    assert rc == -8
    # invalid arguments are reported as by varlen_attn_bwd_v1
    rc = lib.varlen_attn_bwd_noalloc(*(V(args[n]) for n in (
        "dout_ptr", "q_ptr", "k_ptr", "v_ptr", "out_ptr", "lse_ptr", "cu_q_ptr", "cu_k_ptr")),
        2, 10, 10, 5, 5, 8, 2, 96, 1, 0.0, 0, V(0x61000), V(0x62000), V(0x63000), V(0))
    assert rc == -2
    # an empty batch is a no-op that touches nothing
    rc = lib.varlen_attn_bwd_noalloc(*(V(args[n]) for n in (
        "dout_ptr", "q_ptr", "k_ptr", "v_ptr", "out_ptr", "lse_ptr", "cu_q_ptr", "cu_k_ptr")),
        0, 10, 10, 5, 5, 8, 2, 128, 1, 0.0, 0, V(0x61000), V(0x62000), V(0x63000), V(0))
    assert rc == 0


def test_opt_in_status_check_helpers(monkeypatch):
    """The binding's opt-in device status check: the switch and the error it
    raises (no device needed)."""
    import flash_attention_fwd_b200 as fa
    monkeypatch.delenv(fa.STATUS_CHECK_ENV, raising=False)
    assert not fa.status_check_enabled()
    for val, on in (("", False), ("0", False), ("1", True), ("yes", True)):
        monkeypatch.setenv(fa.STATUS_CHECK_ENV, val)
        assert fa.status_check_enabled() == on
    fa.raise_on_status(0)
    with pytest.raises(fa.VarlenAttnError) as err:
        fa.raise_on_status(1)
    assert err.value.code == fa.VARLEN_ERR_DEVICE == -6
    assert "0x1" in str(err.value)
