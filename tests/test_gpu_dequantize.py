"""tq_dequantize vs the oracle's unpacking: value = scale * code of every
coordinate, bit-exact in fp32, and the same fp32 value rounded to nearest even
in bf16 (the layout and scales are those of the tq.h header)."""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import oracle_cache, upload_cache

pytestmark = pytest.mark.gpu


def expected(packed, scales, rows):
    """float32 [B][Hkv][rows][d] = scale[i/32] * code[i] from the oracle's unpack."""
    B, H, cap, half = packed.shape
    d = 2 * half
    codes = oracle.unpack(packed[:, :, :rows].reshape(-1, half), d).astype(np.float32)
    sc = np.repeat(scales[:, :, :rows].reshape(-1, d // 32), 32, axis=1).astype(np.float32)
    return (codes * sc).reshape(B, H, rows, d)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("rows", [1, 37, 300])
def test_dequantize_matches_oracle(d, rows):
    require_cuda()
    B, Hkv, cap = 2, 3, 320
    g = torch.Generator().manual_seed(d + rows)
    k = torch.randn(B, Hkv, cap, d, generator=g)
    v = torch.randn(B, Hkv, cap, d, generator=g) * 3
    signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    cache = oracle_cache(k, v, signs)
    kp, ks, vp, vs = upload_cache(cache)
    for packed_d, scales_d, packed_h, scales_h in ((kp, ks, cache[0], cache[1]), (vp, vs, cache[2], cache[3])):
        want = expected(packed_h, scales_h, rows)
        out32 = torch.empty(B, Hkv, rows, d, dtype=torch.float32, device="cuda")
        _lib.dequantize(packed_d, scales_d, rows, out32)
        out16 = torch.empty(B, Hkv, rows, d, dtype=torch.bfloat16, device="cuda")
        _lib.dequantize(packed_d, scales_d, rows, out16)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out32.cpu().numpy(), want)
        np.testing.assert_array_equal(out16.cpu().view(torch.int16).numpy(),
                                      torch.from_numpy(want).to(torch.bfloat16).view(torch.int16).numpy())
