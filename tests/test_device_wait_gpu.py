"""Bounded on-device waits: a wait that nothing will satisfy runs out, records
FP8Q_ERR_TIMEOUT, and the kernel returns; the context stays usable.  Nothing
faults, traps or hangs."""
import numpy as np
import pytest
import torch

import fp8_fine_grained_quant_b200 as fq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def test_wait_times_out_and_reports(dev):
    assert fq.get_device_error(device=dev) == fq.OK
    fq.selftest_wait_timeout(20_000_000, device=dev)  # 20 ms
    assert fq.get_device_error(device=dev) == fq.ERR_TIMEOUT
    assert fq.get_device_error(device=dev) == fq.OK  # reading clears it


def test_context_usable_after_timeout(dev):
    fq.selftest_wait_timeout(5_000_000, device=dev)
    assert fq.get_device_error(device=dev) == fq.ERR_TIMEOUT
    x = torch.ones((4, 256), dtype=torch.bfloat16, device=dev)
    q, s = fq.fp8_quant_act_1x128(x)
    torch.cuda.synchronize(dev)
    assert torch.all(q.view(torch.uint8) == 0x7E)
    assert fq.get_device_error(device=dev) == fq.OK


def test_launch_counter_counts(dev):
    n0 = fq.launch_count()
    x = torch.ones((4, 256), dtype=torch.bfloat16, device=dev)
    fq.fp8_quant_act_1x128(x)
    assert fq.launch_count() == n0 + 1


def test_set_timeout_roundtrip(dev):
    fq.set_wait_timeout_ns(2_000_000_000)
    fq.set_wait_timeout_ns(0)  # restores the default


@pytest.mark.parametrize("limit_ns", [1_000, 20_000])
@pytest.mark.parametrize("M", [1024, 2048])
def test_gemm_with_a_short_wait_limit_returns_and_recovers(dev, limit_ns, M):
    """A GEMM launched with a wait limit of a few microseconds: waits may run
    out (the call then records FP8Q_ERR_TIMEOUT and the kernel drains its
    copies and MMAs before it frees TMEM and exits) or not (FP8Q_OK); either
    way the call returns, and a GEMM run afterwards with the default limit is
    exact against the oracle.  M = 1024 runs 128 x 128 tiles, M = 2048 the
    128 x 256 tiles (one round of 128 against two)."""
    import oracle
    import workloads as wl
    from parity import assert_gemm_close, bf16_bits_of, to_torch_bf16
    rng = np.random.default_rng(limit_ns + M)
    a = wl.bf16_bits(rng.standard_normal((M, 4096)).astype(np.float32))
    b = wl.bf16_bits((0.02 * rng.standard_normal((2048, 4096))).astype(np.float32))
    qa, sa = fq.fp8_quant_act_1x128(to_torch_bf16(a, dev))
    qb, sb = fq.fp8_quant_w_128x128(to_torch_bf16(b, dev))
    assert fq.get_device_error(device=dev) == fq.OK
    try:
        fq.set_wait_timeout_ns(limit_ns)
        for _ in range(3):
            fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
        st = fq.get_device_error(device=dev)
        assert st in (fq.OK, fq.ERR_TIMEOUT)
    finally:
        fq.set_wait_timeout_ns(0)
    c = fq.fp8_gemm_blockscaled(qa, sa, qb, sb)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    rows = wl.quad_rows(np.random.default_rng(1), M)
    oqa, osa = oracle.quant_act_1x128(a)
    oqb, osb = oracle.quant_w_128x128(b)
    assert_gemm_close(bf16_bits_of(c)[rows], oracle.gemm_blockscaled(oqa, osa, oqb, osb, rows=rows),
                      "after a short wait limit")


def test_masked_gemm_with_a_short_wait_limit_returns(dev):
    rng = np.random.default_rng(3)
    E, cap, N, K = 8, 256, 1024, 2048
    x = torch.from_numpy(rng.standard_normal((E * cap, K)).astype(np.float32)).to(dev).to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((E, N, K))).astype(np.float32)).to(dev).to(torch.bfloat16)
    qa, sa = fq.fp8_quant_act_1x128(x)
    qb, sb = fq.fp8_quant_w_128x128(w)
    mm = torch.tensor([256, 3, 0, 200, 129, 64, 255, 128], dtype=torch.int32, device=dev)
    try:
        fq.set_wait_timeout_ns(1_000)
        fq.fp8_grouped_gemm_masked(qa.view(E, cap, K), sa.view(E, cap, K // 128), qb, sb, mm, expected_m=128)
        assert fq.get_device_error(device=dev) in (fq.OK, fq.ERR_TIMEOUT)
    finally:
        fq.set_wait_timeout_ns(0)
    c = fq.fp8_grouped_gemm_masked(qa.view(E, cap, K), sa.view(E, cap, K // 128), qb, sb, mm, expected_m=128)
    torch.cuda.synchronize(dev)
    assert fq.get_device_error(device=dev) == fq.OK
    assert torch.isfinite(c[0].float()).all()


def test_gemm_rejects_tile_counts_beyond_32_bits(dev):
    """Shapes whose output-tile count does not fit the kernels' 32-bit tile
    numbers are refused before any launch (the pointers are never used: the
    call stops at the tile count, after encoding the tensor maps)."""
    lib = fq.lib()
    fake = 0x10000  # 256-byte aligned, never dereferenced
    big = 1 << 30
    with torch.cuda.device(dev):
        for M, N in ((big, big), (1 << 28, 1 << 24)):
            st = lib.fp8_gemm_blockscaled(fake, fake, fake, fake, fake, M, N, 512, None)
            assert st == fq.ERR_SHAPE, (M, N, st)
    assert fq.get_device_error(device=dev) == fq.OK
