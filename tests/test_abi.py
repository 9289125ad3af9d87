"""The C-ABI library loads, exports every symbol include/fa.h declares, and
rejects bad arguments before it touches the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

import exact_tiled_attention_46_b200 as fa
from exact_tiled_attention_46_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fabuild.build()
    return fa.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_abi_version_and_strings(L):
    assert L.fa_abi_version() == 1
    for code in range(6):
        assert L.fa_status_string(code) and L.fa_status_string(code) != b"unknown status"
    assert L.fa_status_string(99) == b"unknown status"


def test_workspace_sizes(L):
    # decode: o_part [B,Hq,S,D] fp32 + lse_part [B,Hq,S] fp32, each 256-byte aligned
    S = -(-32768 // fa.decode_chunk())
    assert fa.decode_workspace_size(64, 32, 32768, 128) >= 64 * 32 * S * 129 * 4
    # backward: fp32 dQ accumulator + per-row Delta
    assert fa.bwd_workspace_size(8, 16, 4096, 64) >= 8 * 4096 * 16 * 64 * 4 + 8 * 16 * 4096 * 4
    assert fa.bwd_workspace_size(0, 1, 1, 64) == 0


P16 = 4096  # a fake, 16-byte aligned "device" address: never dereferenced on these paths


@pytest.mark.parametrize("args,expect", [
    ((None, P16, P16, P16, None, 1, 1, 1, 8, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),   # null q
    ((P16, None, P16, P16, None, 1, 1, 1, 8, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),   # null k
    ((P16, P16, P16, P16, None, 1, 1, 1, 8, 8, 96, 0.1, 0, None), fa.FA_ERR_UNSUPPORTED),    # D=96
    ((P16, P16, P16, P16, None, 1, 3, 2, 8, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),    # Hq % Hkv
    ((P16 + 2, P16, P16, P16, None, 1, 1, 1, 8, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),  # misaligned
    ((P16, P16, P16, P16, None, 1, 1, 1, 8, 8, 64, -1.0, 0, None), fa.FA_ERR_INVALID_ARG),   # scale <= 0
    ((P16, P16, P16, P16, None, 1, 1, 1, 8, 8, 64, float("nan"), 0, None), fa.FA_ERR_INVALID_ARG),
    ((P16, P16, P16, P16, None, 0, 1, 1, 8, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),    # B = 0
    ((P16, P16, P16, P16, None, 1, 1, 1, -1, 8, 64, 0.1, 0, None), fa.FA_ERR_INVALID_ARG),   # Lq < 0
])
def test_fwd_rejects_bad_arguments(L, args, expect):
    assert L.fa_fwd(*args) == expect


def test_fwd_empty_query_is_noop(L):
    # Lq == 0: valid, nothing to launch
    assert L.fa_fwd(P16, P16, P16, P16, None, 1, 1, 1, 0, 8, 64, 0.1, 0, None) == fa.FA_OK


def test_fwd_ex_bad_dtype(L):
    assert L.fa_fwd_ex(P16, P16, P16, P16, None, 1, 1, 1, 8, 8, 64, 0.1, 0, 7, None) == fa.FA_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(L):
    ws = fa.decode_workspace_size(2, 4, 100, 64)
    ok = (P16, P16, P16, P16, P16, None, 2, 4, 2, 100, 64, 0.1, 0, 256 * 1024, ws)
    bad_ws = ok[:-1] + (ws - 1,)
    assert L.fa_decode_splitkv(*bad_ws, None) == fa.FA_ERR_INVALID_ARG
    bad_align = ok[:13] + (256 * 1024 + 16, ws)
    assert L.fa_decode_splitkv(*bad_align, None) == fa.FA_ERR_INVALID_ARG
    bad_d = ok[:10] + (80,) + ok[11:]
    assert L.fa_decode_splitkv(*bad_d, None) == fa.FA_ERR_UNSUPPORTED
    assert L.fa_decode_combine(None, P16, None, P16, None, 1, 1, 64, 2, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_decode_combine(P16, P16, None, P16, None, 1, 1, 64, 0, 0, None) == fa.FA_ERR_INVALID_ARG


def test_bwd_rejects_bad_arguments(L):
    ws = fa.bwd_workspace_size(1, 2, 128, 64)
    base = [P16] * 9 + [1, 2, 2, 128, 128, 64, 0.125, 1, 0, 256 * 1024, ws, None]
    a = list(base)
    a[19] = ws - 1
    assert L.fa_bwd(*a) == fa.FA_ERR_INVALID_ARG
    a = list(base)
    a[5] = None                       # lse
    assert L.fa_bwd(*a) == fa.FA_ERR_INVALID_ARG
    a = list(base)
    a[14] = 32
    assert L.fa_bwd(*a) == fa.FA_ERR_UNSUPPORTED


def test_selftest_rejects_bad_limit(L):
    assert L.fa_selftest_wait_timeout(0, None) == fa.FA_ERR_INVALID_ARG


def test_binding_has_no_cpu_path():
    import torch
    q = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        fa.fwd(q, q, q)


def test_static_decode_rejects_oversize_before_any_cuda_call(L):
    # 128 sequences x 32 heads x 32 chunks of partials exceed the file-scope array
    assert fa.decode_workspace_size(128, 32, 32768, 128) > 40 * 1024 * 1024
    assert L.fa_decode_splitkv_static(P16, P16, P16, P16, P16, None, 128, 32, 8, 32768, 128, 0.1, 0,
                                      None) == fa.FA_ERR_UNSUPPORTED


def test_bwd_rejects_dtype_and_workspace_alignment(L):
    ws = fa.bwd_workspace_size(1, 2, 128, 64)
    base = [P16] * 9 + [1, 2, 2, 128, 128, 64, 0.125, 1, 0, 256 * 1024, ws, None]
    a = list(base)
    a[17] = 7                          # grad dtype
    assert L.fa_bwd(*a) == fa.FA_ERR_INVALID_ARG
    a = list(base)
    a[18] = 256 * 1024 + 16            # workspace only 16-byte aligned
    assert L.fa_bwd(*a) == fa.FA_ERR_INVALID_ARG
    a = list(base)
    a[5] = P16 + 2                     # lse not 4-byte aligned
    assert L.fa_bwd(*a) == fa.FA_ERR_INVALID_ARG


def test_fwd_rejects_misaligned_lse(L):
    assert L.fa_fwd(P16, P16, P16, P16, P16 + 2, 1, 1, 1, 8, 8, 64, 0.1, 0, None) == fa.FA_ERR_INVALID_ARG


def test_exp2_selftest_rejects_bad_arguments(L):
    assert L.fa_selftest_exp2_poly(None, P16, 4, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_selftest_exp2_poly(P16, P16, -1, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_selftest_exp2_poly(P16, P16, 0, None) == fa.FA_OK      # nothing to launch


def test_launch_guard_reports_per_instantiation_state_without_gpu(L):
    """Before any launch every kernel instantiation's register check result is
    'not yet checked'; querying it (without the compiled count, which needs a
    GPU) changes nothing."""
    for bwd in (0, 1):
        for D in (64, 128):
            for causal in (0, 1):
                regs, expected, state = fa.launch_guard(bwd, D, causal, query_regs=False)
                assert regs is None and state == 0
                assert expected == (128 if bwd else 168)
    st = L.fa_launch_guard(0, 96, 0, None, None, None)
    assert st == fa.FA_ERR_INVALID_ARG


def test_decode_append_rejects_bad_arguments(L):
    # q, k_new, v_new, k_cache, v_cache, seqlens, o, lse, B, Hq, Hkv, Lmax, D, scale, o_dtype, ws, bytes, stream
    ws = fa.decode_workspace_size(2, 4, 101, 64)
    ok = [P16] * 7 + [None, 2, 4, 2, 100, 64, 0.1, 0, 256 * 1024, ws, None]
    a = list(ok)
    a[16] = fa.decode_workspace_size(2, 4, 100, 64) - 1   # too small for Lmax + 1 keys
    assert L.fa_decode_append_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[1] = None                                            # k_new
    assert L.fa_decode_append_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[2] = P16 + 8                                         # v_new misaligned
    assert L.fa_decode_append_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[12] = 96
    assert L.fa_decode_append_splitkv(*a) == fa.FA_ERR_UNSUPPORTED


def test_decode_paged_rejects_bad_arguments(L):
    # q, k_new, v_new, k_pages, v_pages, table, seqlens, o, lse, B, Hq, Hkv, num_pages, page, pps, D, scale,
    # o_dtype, ws, bytes, stream
    ws = fa.decode_workspace_size(2, 4, 4 * 256, 64)     # capacity 1024 rows: one chunk, two with an append
    ok = [P16, None, None, P16, P16, P16, P16, P16, None, 2, 4, 2, 10, 256, 4, 64, 0.1, 0, 256 * 1024, ws, None]
    a = list(ok)
    a[13] = 24                                             # page size not a multiple of 16
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_UNSUPPORTED
    a = list(ok)
    a[5] = None                                            # no page table
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[1] = P16                                             # k_new without v_new
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[1], a[2] = P16, P16                                  # append needs one more key of workspace
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[5] = P16 + 2                                         # misaligned table
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[12] = 0                                              # empty pool
    assert L.fa_decode_paged_splitkv(*a) == fa.FA_ERR_INVALID_ARG


def test_fwd_fp8_rejects_bad_arguments(L):
    # q, k, v, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, o_dtype, stream
    ok = [P16, P16, P16, 1.0, 1.0, 1.0, P16, None, 1, 2, 2, 8, 8, 128, 0.1, 1, 0, None]
    a = list(ok)
    a[13] = 64
    assert L.fa_fwd_fp8(*a) == fa.FA_ERR_UNSUPPORTED
    for i in (3, 4, 5):
        a = list(ok)
        a[i] = 0.0                                          # scales must be > 0
        assert L.fa_fwd_fp8(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[1] = P16 + 8
    assert L.fa_fwd_fp8(*a) == fa.FA_ERR_INVALID_ARG


def test_attn_merge_rejects_bad_arguments(L):
    # o_a, lse_a, o_b, lse_b, o_out, lse_out, B, H, L, D, o_dtype, stream
    ok = [P16] * 6 + [1, 2, 8, 128, 1, None]
    a = list(ok)
    a[9] = 126                                             # D not a multiple of 4
    assert L.fa_attn_merge(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[2] = None
    assert L.fa_attn_merge(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[1] = P16 + 2
    assert L.fa_attn_merge(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok)
    a[8] = 0                                               # nothing to merge
    assert L.fa_attn_merge(*a) == fa.FA_OK


def test_debug_build_compiles_exports_and_reports_itself(L):
    """The FA_DEBUG build (index checks on every global store) builds from the
    same sources, exports the same symbols and says which build it is."""
    path = fabuild.build(debug=True)
    D = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(D, n), n
    D.fa_status_string.restype = ctypes.c_char_p
    assert D.fa_debug_build() == 1 and L.fa_debug_build() == 0
    assert D.fa_status_string(fa.FA_ERR_DEVICE_INDEX) == b"device index check failed (debug build)"
