"""The seeded input generator (msa_inputs) against its published definition: SplitMix64's
reference outputs, the tensor form equal to the integer form, Box-Muller normals, element
values independent of how a tensor is chunked, and one rounding to bf16."""
import numpy as np
import torch

import msa_inputs as mi


def test_splitmix64_reference_outputs_seed_zero():
    # SplitMix64 seeded with 0: the generator's widely published first four outputs
    state, outs = 0, []
    for _ in range(4):
        state = (state + mi._GAMMA) & mi._MASK64
        outs.append(mi._mix64_int(state))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F,
                    0xF88BB8A8724C81EC]


def test_tensor_mixer_equals_integer_mixer():
    rng = np.random.default_rng(0)
    vals = [int(x) for x in rng.integers(0, 2**63, 64, dtype=np.uint64)] + [0, 2**64 - 1, 2**63]
    t = torch.tensor([mi._signed(v) for v in vals], dtype=torch.int64)
    got = [int(x) & mi._MASK64 for x in mi._mix64_t(t)]
    assert got == [mi._mix64_int(v) for v in vals]


def test_normal_moments_and_independence_of_streams():
    a = mi.normal((1 << 20,), seed=0, stream=1, dtype=torch.float64)
    b = mi.normal((1 << 20,), seed=0, stream=2, dtype=torch.float64)
    for x in (a, b):
        assert abs(float(x.mean())) < 5e-3
        assert abs(float(x.var()) - 1.0) < 5e-3
        assert abs(float((x ** 4).mean()) - 3.0) < 3e-2         # Gaussian kurtosis
    assert abs(float((a * b).mean())) < 5e-3                     # streams uncorrelated


def test_elements_do_not_depend_on_chunking():
    base = mi.stream_base(7, mi.STREAM_K)
    whole = mi._normal_chunk(base, 0, 5000, "cpu")
    idx = torch.tensor([4999, 0, 1234, 17, 4096])
    np.testing.assert_array_equal(mi._normal_idx(base, idx).numpy(), whole[idx].numpy())
    part = mi._normal_chunk(base, 1000, 2000, "cpu")
    np.testing.assert_array_equal(part.numpy(), whole[1000:3000].numpy())


def test_bf16_tensor_is_one_rounding_of_the_fp32_tensor():
    x32 = mi.normal((4096,), seed=3, stream=1, dtype=torch.float32)
    x16 = mi.normal((4096,), seed=3, stream=1, dtype=torch.bfloat16)
    assert torch.equal(x32.to(torch.bfloat16), x16)


def test_rows_of_a_tensor_generate_alone():
    """A shard's rows of a bank, generated on their own, are the full tensor's rows."""
    full = mi.normal((300, 3, 8), 5, mi.STREAM_K, "cpu", torch.bfloat16)
    for lo, hi in [(0, 300), (17, 18), (100, 299), (0, 1)]:
        part = mi.normal_rows((300, 3, 8), lo, hi, 5, mi.STREAM_K, "cpu", torch.bfloat16)
        assert torch.equal(part, full[lo:hi])
    w = mi.Workload("b", "decode", 1, 500, 8, 2, 16, 16, 4, "bf16", n_query=2)
    _, k, v = mi.decode_inputs(w, seed=1)
    k2, v2 = mi.decode_bank_rows(w, 123, 456, seed=1)
    assert torch.equal(k2, k[123:456]) and torch.equal(v2, v[123:456])
