"""The decode entry point that allocates nothing (fa_decode_splitkv_static).

Some callers cannot allocate device memory when they run a decode step (an
engine plugin or serving loop with memory fixed at start-up, where cudaMalloc
could block and synchronise the device; a foreign caller that only owns its
tensors).  This entry point keeps its partial results in a fixed array inside
the library instead of a caller workspace.  Its output must match the regular
entry point (which takes a workspace) within the tolerances of the other parity
tests, on two calls in a row with different problems, so that the second call
cannot be helped or hurt by what the first left in the shared array.  The file
is named to be collected last.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_tiled_attention_46_b200 as fa
from exact_tiled_attention_46_b200 import inputs as synth

from parity import check_close, check_lse, need_gpu, f64

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 40 * 1024 * 1024   # FA_DECODE_STATIC_SCRATCH_BYTES in include/fa.h


def call_static(q, kc, vc, sl, out, lse, scale):
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = kc.shape
    odt = 1 if out.dtype == torch.float32 else 0
    return fa.lib().fa_decode_splitkv_static(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(),
                                             out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lmax, D, scale, odt,
                                             torch.cuda.current_stream().cuda_stream)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def test_no_alloc_decode_matches_regular_on_two_calls():
    problems = [
        # B, Hq, Hkv, Lmax, D, lengths, seed
        (6, 32, 8, 5000, 128, [4999, 1, 1024, 1025, 3000, 5000], 11),
        (3, 8, 2, 2100, 64, [2100, 17, 700], 12),
    ]
    for B, Hq, Hkv, Lmax, D, lens, seed in problems:
        assert fa.decode_workspace_size(B, Hq, Lmax, D) <= SCRATCH_BYTES
        x = synth.decode_inputs(B, Hq, Hkv, Lmax, D, seed, 1, Lmax, lens=lens, pad_value=float("nan"))
        q, kc, vc, sl = x["q"].cuda(), x["k_cache"].cuda(), x["v_cache"].cuda(), x["seqlens"].cuda()
        scale = 1.0 / math.sqrt(D)
        ref_o, ref_l = fa.decode(q, kc, vc, sl, scale=scale, o_dtype=torch.float32)
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        assert call_static(q, kc, vc, sl, out, lse, scale) == fa.FA_OK
        torch.cuda.synchronize()
        check_close(f64(out), f64(ref_o), bf16_output=False, what="no-alloc O")
        check_lse(f64(lse), f64(ref_l), what="no-alloc LSE")
        # and against the CPU fp64 oracle directly
        ro, rl = oracle.attn_decode(synth.as_f64(x["q"]), synth.as_f64(x["k_cache"]), synth.as_f64(x["v_cache"]),
                                    x["seqlens"].numpy(), scale)
        check_close(f64(out), ro, bf16_output=False, what="no-alloc O vs oracle")
        check_lse(f64(lse), rl, what="no-alloc LSE vs oracle")


def test_no_alloc_decode_rejects_configurations_beyond_the_scratch():
    # 64 sequences x 32 heads with a 65536-row cache need ~68 MB of partials
    B, Hq, Hkv, Lmax, D = 64, 32, 8, 65536, 128
    assert fa.decode_workspace_size(B, Hq, Lmax, D) > SCRATCH_BYTES
    p16 = 1 << 20    # never dereferenced: the call returns before any launch
    st = fa.lib().fa_decode_splitkv_static(p16, p16, p16, p16, p16, p16, B, Hq, Hkv, Lmax, D, 0.1, 0, None)
    assert st == fa.FA_ERR_UNSUPPORTED
