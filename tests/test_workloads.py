"""The seeded input recipe: deterministic, bf16, with the stated structure."""
import torch

from io_aware_exact_32_b200 import workloads as W


def test_attention_inputs_deterministic_and_bf16():
    a = W.make_attention_inputs(1, 2, 33, 47, 64, seed=5)
    b = W.make_attention_inputs(1, 2, 33, 47, 64, seed=5)
    for n in ("q", "k", "v", "do"):
        assert a[n].dtype == torch.bfloat16
        assert torch.equal(a[n], b[n])
    assert a["q"].shape == (1, 2, 33, 64) and a["k"].shape == (1, 2, 47, 64)
    c = W.make_attention_inputs(1, 2, 33, 47, 64, seed=6)
    assert not torch.equal(a["q"], c["q"])


def test_peaked_keys_exact_times_eight():
    base = W.make_attention_inputs(2, 2, 16, 400, 64, seed=7)
    pk = W.make_attention_inputs(2, 2, 16, 400, 64, seed=7, peaked_frac=0.01)
    assert pk["peaks"].shape == (2, 2, 4)
    for b in range(2):
        for h in range(2):
            idx = pk["peaks"][b, h]
            assert len(set(idx.tolist())) == 4
            assert torch.equal(pk["k"][b, h, idx].float(), base["k"][b, h, idx].float() * 8)
            mask = torch.ones(400, dtype=torch.bool)
            mask[idx] = False
            assert torch.equal(pk["k"][b, h, mask], base["k"][b, h, mask])
    assert torch.equal(pk["q"], base["q"]) and torch.equal(pk["v"], base["v"])


def test_decode_inputs():
    x = W.make_decode_inputs(32, 2, 8192, 128, 1024, seed=4)
    L = x["seqlens"]
    assert L.dtype == torch.int32 and L.shape == (32,)
    assert int(L.min()) >= 1024 and int(L.max()) <= 8192
    assert x["k_cache"].shape == (32, 2, 8192, 128) and x["q"].shape == (32, 2, 1, 128)


def test_flop_and_byte_conventions():
    assert W.flops_forward(2, 8, 1024, 1024, 64, False) == 4.0 * 2 * 8 * 1024 * 1024 * 64
    assert W.flops_forward(2, 8, 1024, 1024, 64, True) == 2.0 * 2 * 8 * 1024 * 1024 * 64
    assert W.flops_backward(1, 1, 4, 4, 2, False) == 2.5 * 4 * 16 * 2
    assert W.decode_bytes(torch.tensor([3, 5]), 2, 4) == 8 * 2 * 4 * 2 * 2 + 2 * 2 * 2 * 4 * 2


def test_config_table():
    assert W.TINY.B == 1 and W.TINY.H == 2 and W.TINY.Nq == 128 and W.TINY.d == 64
    assert [c.Nq * c.B for c in W.SWEEP] == [16384] * 12
    assert {c.d for c in W.SWEEP} == {64, 128}
    assert W.LONG.Nq == 65536 and W.LONG.peaked_frac == 0.01
    assert W.DECODE.B == 32 and W.DECODE.H == 32 and W.DECODE.Lmax == 8192
