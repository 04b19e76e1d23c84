"""The seeded input generator (CPU only)."""
import numpy as np
import torch

from exact_tiled_attention_32_b200 import synthetic as syn


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = rng.normal(0, 3, 100000).astype(np.float32).astype(np.float64)
    x = np.concatenate([x, [0.0, -0.0, 1.0, 65504.0, 1e-30, -3.5]])
    ours = syn.fp64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, ref.view(np.uint16))


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: even is 1
    assert syn.fp64_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert syn.fp64_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82
    # just above the halfway point rounds up
    assert syn.fp64_to_bf16_bits(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81


def test_stream_is_counter_based_and_deterministic():
    a = syn.splitmix64(5, 0, 1000)
    b = np.concatenate([syn.splitmix64(5, 0, 400), syn.splitmix64(5, 400, 600)])
    assert np.array_equal(a, b)
    s1, s2 = syn.Stream(9), syn.Stream(9)
    assert np.array_equal(s1.normal_bf16((3, 5)), s2.normal_bf16((3, 5)))
    # threaded and single-threaded generation agree
    big1 = syn.Stream(1).normal_bf16((1 << 23) + 3, threads=8)
    big2 = syn.Stream(1).normal_bf16((1 << 23) + 3, threads=1)
    assert np.array_equal(big1, big2)


def test_normals_look_normal():
    z = syn.bf16_bits_to_float(syn.Stream(3).normal_bf16(200000)).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    assert abs(np.mean(np.abs(z) < 1.0) - 0.6827) < 0.005


def test_workloads():
    c5 = syn.config("c5")
    assert len(c5.seqlens) == 16 and all(512 <= L <= 8192 for L in c5.seqlens)
    assert c5.cu_seqlens[-1] == c5.N and c5.cu_seqlens.dtype == np.int32
    assert syn.config("c3").flops() == 4 * 16384 ** 2 * 128 * 32 / 2
    assert syn.config("c1").flops() == 4 * 256 ** 2 * 64
    # the pages' closed forms for the size of S in FP16 (one batch, one head):
    # 8 GiB at N = 64K and 2 GiB at N = 32K
    assert 65536 ** 2 * 2 == 8 * 2 ** 30 and 32768 ** 2 * 2 == 2 * 2 ** 30
    w = syn.config("c1").draw()
    assert w.q.shape == (1, 1, 256, 64) and w.q.dtype == np.uint16
    w2 = syn.config("c1").draw()
    assert np.array_equal(w.v, w2.v)
