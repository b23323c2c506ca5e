"""Cases for tests/test_gpu_tail.py, which runs them in a child process with
256-column tiles forced (the planner picks 128 for these small shapes, and
only 256-wide dense tiles split their tail).

Dense split-K tail: the partial last wave's tiles run as a second launch that
splits each along K over a cluster of 2, 4 or 8 CTAs, which sum their FP32
partials through distributed shared memory. Capping the grid with
dg_set_num_sms makes small shapes have a tail: the whole output is compared
with the oracle, and repeated runs must agree bit for bit (the parts are
summed in a fixed order).
"""
import numpy as np
import pytest
import torch

import moe_grouped_gemm_07_b200 as dg
import oracle
import synth
import synth.workloads as wl
from gpu_helpers import as_f64, bf16_dev, check_close, dev, to_dev

pytestmark = pytest.mark.gpu

# (M, N, K, grid cap, with C): tiles = ceil(M/128) * ceil(N/256); a split must
# save >= 40 K-blocks per tile, hence the long K
CASES = [
    (384, 768, 8192, 8, True),      # 9 tiles on 8 CTAs: 1 tail tile x 4 parts
    (256, 512, 12288, 3, False),    # 4 tiles on 3: 1 x 2 parts
    (2176, 256, 8192, 16, False),   # 17 tiles on 16: 1 x 8 parts
    (600, 1000, 12288, 16, True),   # ragged M and N: 4 tail tiles x 4 parts
    (896, 512, 512, 12, False),     # 14 tiles on 12: too short to split (plain last wave)
]


@pytest.mark.parametrize("M,N,K,sms,with_c", CASES)
def test_split_tail_vs_oracle(M, N, K, sms, with_c):
    w = wl.dense(M, N, K, cfg=96, shape=M + N + K + sms, with_c=with_c)
    Cb = synth.to_bf16_bits(w.C) if with_c else None
    qa, sa = dg.dg_quantize_fp8(to_dev(w.A), dg.DG_QUANT_ROW_1x128)
    qb, sb = dg.dg_quantize_fp8(to_dev(w.B), dg.DG_QUANT_BLOCK_128x128)
    R = oracle.gemm_nt(*oracle.quantize(w.A, oracle.ROW_1x128), *oracle.quantize(w.B, oracle.BLOCK_128x128), Cb)
    dg.dg_set_num_sms(sms)
    try:
        outs = []
        for _ in range(3):
            D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev())
            dg.dg_fp8_gemm_nt(qa, sa, qb, sb, bf16_dev(Cb) if with_c else None, D)
            outs.append(D)
        assert dg.dg_get_last_device_error() == (dg.DG_OK, 0)
    finally:
        dg.dg_set_num_sms(0)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    check_close(as_f64(outs[0]), R, f"split tail {M}x{N}x{K} on {sms} CTAs")
    # the same problem without a tail (all SMs) gives the same result within tolerance
    D2 = torch.empty((M, N), dtype=torch.bfloat16, device=dev())
    dg.dg_fp8_gemm_nt(qa, sa, qb, sb, bf16_dev(Cb) if with_c else None, D2)
    check_close(as_f64(D2), R, "no tail")
