"""GPU parity of the FP8 (E4M3) paged decode (fa_decode_paged_fp8) against
the fp64 oracle over the same FP8 codes and scales, through the C ABI.
Same tolerances as the bf16 decode (tests/parity.py): the codes are exact
inputs, so only the kernel's fp32 arithmetic and the bf16 output differ."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def run(fa, w, sinks=None):
    o, lse = fa.decode_paged_fp8(w.q.cuda(), w.k_codes.cuda(), w.v_codes.cuda(),
                                 w.k_scale.cuda(), w.v_scale.cuda(), w.block_table.cuda(),
                                 w.seq_lens.cuda(), w.scale,
                                 sinks=None if sinks is None else sinks.cuda())
    assert fa.check_device_error() == 0
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 2), (6, 3), (16, 4), (12, 4), (32, 1)])
def test_fp8_shapes(fa, d, Hq, Hkv):
    """Group sizes 1, 2, 4 and 8 run on the tensor-core kernel with 1, 2, 4 or 8
    pages per tile (eight, four, two or one KV heads per unit); 3 and 32 on the
    CUDA-core kernel."""
    w = workloads.paged_fp8(lens=[1, 15, 16, 17, 255, 256, 257, 1000], Hq=Hq, Hkv=Hkv, d=d,
                            seed=Hq + d, poison=True, spare_pages=3)
    o, lse = run(fa, w)
    o_ref, lse_ref = oracle.decode_paged_fp8(w.q, w.k_codes, w.v_codes, w.k_scale, w.v_scale,
                                             w.block_table, w.seq_lens, w.scale)
    compare(o, o_ref, lse, lse_ref, f"fp8 Hq={Hq} Hkv={Hkv} d={d}")


def test_fp8_sinks_and_empty(fa):
    w = workloads.paged_fp8(lens=[0, 33, 4097], Hq=32, Hkv=8, d=128, seed=2)
    g = torch.Generator("cpu").manual_seed(2)
    z = torch.randn(32, generator=g) * 2.0
    z[3] = -math.inf
    o, lse = run(fa, w, z)
    o_ref, lse_ref = oracle.decode_paged_fp8(w.q, w.k_codes, w.v_codes, w.k_scale, w.v_scale,
                                             w.block_table, w.seq_lens, w.scale,
                                             sinks=z.double().numpy())
    compare(o, o_ref, lse, lse_ref, "fp8 sinks")


def test_fp8_pow2_equals_bf16_kernel(fa):
    """With power-of-two scales the dequantised cache is exactly bf16; the FP8
    kernel and the bf16 kernel then attend to the same values."""
    w = workloads.paged_fp8(pow2_scales=True, lens=[100, 2000, 513], Hq=32, Hkv=8, d=128,
                            seed=8)
    kb = (w.k_codes.view(torch.float8_e4m3fn).float() * w.k_scale[:, None, :, None]).bfloat16()
    vb = (w.v_codes.view(torch.float8_e4m3fn).float() * w.v_scale[:, None, :, None]).bfloat16()
    o8, l8 = run(fa, w)
    ob, lb = fa.decode_paged(w.q.cuda(), kb.cuda(), vb.cuda(), w.block_table.cuda(),
                             w.seq_lens.cuda(), w.scale)
    assert (o8.float() - ob.float()).abs().max().item() <= 1e-2
    assert (l8 - lb).abs().max().item() <= 1e-4


def test_fp8_decode64_full(fa):
    """The decode64 workload (64 sequences, 4,096-32,768 tokens, Hq=32, Hkv=8,
    d=128, seed 0) with its cache in FP8: sampled sequences against the oracle."""
    w = workloads.paged_fp8(**{k: v for k, v in workloads.CONFIGS["decode64"].items()
                               if k != "kind"}, seed=0)
    o, lse = run(fa, w)
    idx = [0, 1, 17, 63]
    o_ref, lse_ref = oracle.decode_paged_fp8(w.q[idx], w.k_codes, w.v_codes, w.k_scale,
                                             w.v_scale, w.block_table[idx], w.seq_lens[idx],
                                             w.scale)
    compare(o[idx], o_ref, lse[idx], lse_ref, "fp8 decode64")
