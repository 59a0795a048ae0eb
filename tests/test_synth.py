"""The seeded input generator: Philox4x32-10 known-answer vectors (Salmon et al.,
SC'11, as published with the Random123 library), slice regeneration and the
value recipe of the workloads."""
import torch

from attention_learned_relative_b200 import synth
from attention_learned_relative_b200.workloads import WORKLOADS, make_inputs


def _philox(ctr, key):
    t = [torch.tensor([c], dtype=torch.int64) for c in ctr]
    return ["%08x" % int(x) for x in synth.philox4x32_10(*t, key[0], key[1])]


def test_philox_known_answers():
    assert _philox([0, 0, 0, 0], [0, 0]) == ["6627e8d5", "e169c58d", "bc57ac4c", "9b00dbd8"]
    assert _philox([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2) == ["408f276d", "41c83b0e", "a20bc7c6", "6d5451fd"]
    assert _philox([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0]) == \
        ["d16cfe09", "94fdcceb", "5001e420", "24126ea1"]


def test_slices_regenerate_exactly():
    full = synth.normal((3, 1001), 7, "k", std=0.5, dtype=torch.float32, chunk=257)
    idx = torch.tensor([0, 1, 2, 3, 4, 1000, 1001, 2999, 3002, 1500])
    part = synth.normal_slice((3, 1001), 7, "k", idx, std=0.5, dtype=torch.float32)
    assert torch.equal(full.reshape(-1)[idx], part)


def test_streams_differ_and_look_normal():
    a = synth.normal((200000,), 1, "q", dtype=torch.float64)
    b = synth.normal((200000,), 1, "k", dtype=torch.float64)
    c = synth.normal((200000,), 2, "q", dtype=torch.float64)
    assert not torch.equal(a, b) and not torch.equal(a, c)
    assert abs(a.mean().item()) < 0.01 and abs(a.std().item() - 1.0) < 0.01
    assert abs(torch.corrcoef(torch.stack([a, b]))[0, 1].item()) < 0.01


def test_workload_recipe():
    wl = WORKLOADS["local_prefill_bf16"]
    x = make_inputs(wl, T=64, B=1)
    assert x["q"].dtype == torch.bfloat16 and x["q"].shape == (1, 64, 32, 128)
    assert x["k"].shape == (1, 64, 4, 128) and x["r"].shape == (1, 64, 32)
    assert x["w"].shape == (32, 512) and x["w"].dtype == torch.float32
    assert abs(x["w"].std().item() - 0.5) < 0.02
    wl4 = WORKLOADS["global_long_prefill_bf16"]
    y = make_inputs(wl4, T=256, B=1)
    assert abs(y["q"].float().std().item() - 0.5) < 0.02
    assert abs(y["v"].float().std().item() - 1.0) < 0.03
