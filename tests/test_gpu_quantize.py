"""GPU quantize-append vs the oracle on the same inputs.

Bar: rotation off -> packed bytes and scales bit-identical; rotation on ->
at most 0.01% of codes differ, each by exactly 1, scales within 4 ulp."""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_tq_b200 import _lib
from conftest import require_cuda
from helpers import oracle_cache, to_oracle

pytestmark = pytest.mark.gpu


def inputs(B, H, n, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, H, n, d, generator=g)
    v = torch.randn(B, H, n, d, generator=g)
    # structure: per-row magnitudes over 8 decades, outlier channels, zero rows
    k *= torch.exp(torch.empty(B, H, n, 1).uniform_(-8, 8, generator=g))
    v *= torch.exp(torch.empty(B, H, n, 1).uniform_(-8, 8, generator=g))
    k[..., 3] *= 10
    if n > 2:
        k[:, :, 1] = 0
        v[:, :, 2] = 0
    return k.to(dtype), v.to(dtype)


def run_gpu(k, v, pos, signs, cap):
    B, H, n, d = k.shape
    dev = "cuda"
    kp = torch.zeros(B, H, cap, d // 2, dtype=torch.uint8, device=dev)
    vp = torch.zeros_like(kp)
    ks = torch.zeros(B, H, cap, d // 32, dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    _lib.quantize_append(k.to(dev), v.to(dev), torch.tensor(pos, dtype=torch.int32, device=dev),
                         None if signs is None else signs.to(dev), kp, ks, vp, vs)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (kp, ks, vp, vs)]


def compare(gpu, ref, d, rot, label, max_scale_ulp=4):
    kp, ks, vp, vs = gpu
    rkp, rks, rvp, rvs = ref
    if not rot:
        np.testing.assert_array_equal(kp, rkp, err_msg=label)
        np.testing.assert_array_equal(vp, rvp, err_msg=label)
        np.testing.assert_array_equal(ks.view(np.uint32), rks.view(np.uint32), err_msg=label)
        np.testing.assert_array_equal(vs.view(np.uint32), rvs.view(np.uint32), err_msg=label)
        return 0, 0
    n_diff, n_tot = 0, 0
    for a, b in ((kp, rkp), (vp, rvp)):
        ca = oracle.unpack(a.reshape(-1, d // 2), d).astype(np.int64)
        cb = oracle.unpack(b.reshape(-1, d // 2), d).astype(np.int64)
        diff = np.abs(ca - cb)
        assert diff.max() <= 1, label
        n_diff += int((diff > 0).sum())
        n_tot += diff.size
    assert n_diff <= 1e-4 * n_tot, f"{label}: {n_diff}/{n_tot} codes differ"
    for a, b in ((ks, rks), (vs, rvs)):
        ulp = np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))
        assert ulp.max() <= max_scale_ulp, f"{label}: scale ulp {ulp.max()}"
    return n_diff, n_tot


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rot", [False, True])
@pytest.mark.parametrize("B,H,n", [(1, 1, 1), (2, 3, 33), (1, 8, 257), (3, 2, 1000), (1, 3, 2999)])
def test_quantize_matches_oracle(d, dtype, rot, B, H, n):
    require_cuda()
    seed = d + n + B * 7 + (1 if rot else 0)
    k, v = inputs(B, H, n, d, dtype, seed)
    cap = n + 9
    pos = [(3 * b) % 10 for b in range(B)]
    signs = None
    if rot:
        g = torch.Generator().manual_seed(seed + 99)
        signs = (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.int8)
    ref = oracle_cache(k, v, signs, capacity=cap, pos=pos)
    gpu = run_gpu(k, v, pos, signs, cap)
    compare(gpu, ref, d, rot, f"d={d} {dtype} rot={rot} B={B} H={H} n={n}")


@pytest.mark.parametrize("d", [128, 256])
def test_quantize_hand_ties_and_extremes_bit_exact(d):
    """Round-half-even ties, all-zero groups, subnormal and huge scales."""
    require_cuda()
    from test_oracle_pins import _read_ties
    groups = _read_ties()
    row = np.concatenate([g[1] for g in groups] * (d // 128))
    rows = [row, -row, np.zeros(d), np.full(d, 1e-40), np.full(d, 3e-39) * np.sign(np.arange(d) - 60.5),
            np.linspace(-1e30, 2e30, d), np.linspace(-7, 7, d) * 2.0 ** -130]
    x = torch.tensor(np.stack(rows), dtype=torch.float32).reshape(1, 1, len(rows), d)
    ref = oracle_cache(x, x, None)
    gpu = run_gpu(x, x, [0], None, len(rows))
    compare(gpu, ref, d, False, "ties/extremes")
    # the tie row's GPU codes are the hand-derived round-half-even codes
    codes = oracle.unpack(gpu[0][0, 0, :1], d)[0].astype(np.int64)
    want = np.concatenate([g[2] for g in groups] * (d // 128))
    np.testing.assert_array_equal(codes, want)


def test_quantize_leaves_other_rows_and_skips_out_of_range():
    require_cuda()
    d, H, n, cap = 128, 2, 4, 8
    k, v = inputs(2, H, n, d, torch.bfloat16, 5)
    dev = "cuda"
    kp = torch.full((2, H, cap, d // 2), 0xAB, dtype=torch.uint8, device=dev)
    vp = kp.clone()
    ks = torch.full((2, H, cap, d // 32), -1.0, device=dev)
    vs = ks.clone()
    pos = torch.tensor([6, 2], dtype=torch.int32, device=dev)   # b=0 overflows after 2 rows
    _lib.quantize_append(k.to(dev), v.to(dev), pos, None, kp, ks, vp, vs)
    torch.cuda.synchronize()
    ref = oracle_cache(k, v, None, capacity=cap + n, pos=[6, 2])
    kp, ks = kp.cpu().numpy(), ks.cpu().numpy()
    np.testing.assert_array_equal(kp[0, :, 6:8], ref[0][0, :, 6:8])
    assert np.all(kp[0, :, :6] == 0xAB) and np.all(ks[0, :, :6] == -1.0)
    np.testing.assert_array_equal(kp[1, :, 2:6], ref[0][1, :, 2:6])
    assert np.all(kp[1, :, :2] == 0xAB) and np.all(kp[1, :, 6:] == 0xAB)


def test_quantize_rejects_bad_args_without_launch():
    require_cuda()
    d = 128
    x = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(1, 1, 4, 32, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, 1, 4, 2, device="cuda")
    p = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.TQError) as e:
        _lib.quantize_append(x, x, p, None, c, s, c, s)
    assert e.value.status == _lib.TQ_ERR_UNSUPPORTED
    assert d == 128
