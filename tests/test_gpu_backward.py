"""GPU parity of the backward pass (relbias_attn_bwd) against the fp64 oracle's
gradients (oracle_attn_bwd, itself pinned by finite differences of the forward).

bf16 inputs with d in {64, 128} run on the tcgen05 kernels (backward_sm100.cu), fp32
and other head sizes on the CUDA-core kernels (backward_fp32.cu).
The kernel gets O and LSE from the oracle's forward (stored in the kernel's dtype),
as a training step would get them from the forward pass.  Tolerance, relative to the
largest reference gradient of each tensor: 1e-4 for fp32 (fp32 sums of up to a few
thousand terms); 1e-2 for bf16, where O is stored in bf16 and D_i = dout_i . o_i
inherits its 2^-9 relative rounding.
"""
import math

import pytest
import torch

from attention_learned_relative_b200 import ops, synth
from oracle import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    ops.device_status(reset=True)
    yield
    assert ops.device_status(reset=True) == 0, "a kernel wait timed out"


def _inputs(dtype, B, T, Hq, Hkv, d, R, seed):
    dev = "cuda"
    return {
        "q": synth.normal((B, T, Hq, d), seed, "q", dtype=dtype, device=dev),
        "k": synth.normal((B, T, Hkv, d), seed, "k", dtype=dtype, device=dev),
        "v": synth.normal((B, T, Hkv, d), seed, "v", dtype=dtype, device=dev),
        "r": synth.normal((B, T, Hq), seed, "r", device=dev),
        "w": synth.normal((Hq, R), seed, "w", std=0.5, device=dev),
        "dout": synth.normal((B, T, Hq, d), seed, "bank", dtype=dtype, device=dev),
    }


def _check(g, ref, tol, what):
    for name in ("dq", "dk", "dv", "dr", "dw"):
        a = g[name].double().cpu()
        b = torch.as_tensor(ref[name]).reshape(a.shape)
        if b.numel() == 0:
            continue
        scale = b.abs().max().item()
        err = (a - b).abs().max().item()
        assert err <= tol * scale + 1e-7, "%s %s: max err %.3e vs max |ref| %.3e" % (what, name, err, scale)


CASES = [
    # dtype,          B, T,    Hq, Hkv, d,   window, R,   temp_n0
    (torch.float32, 1, 100, 4, 2, 64, 0, 50, 0),
    (torch.float32, 2, 150, 4, 1, 32, 40, 60, 0),       # window, GQA group 4, ragged tiles
    (torch.float32, 1, 300, 2, 2, 128, 0, 300, 100),    # temperature
    (torch.float32, 1, 97, 4, 4, 256, 16, 20, 0),       # d = 256
    (torch.float32, 1, 64, 2, 1, 64, 0, 0, 0),          # R = 0: no bias, no dw
    (torch.bfloat16, 1, 256, 8, 2, 128, 0, 128, 0),
    (torch.bfloat16, 1, 1024, 8, 2, 128, 512, 512, 0),  # the local-layer shape over 32 tiles
    (torch.bfloat16, 1, 300, 6, 2, 64, 0, 100, 0),      # d = 64, group 3, ragged last tile
    (torch.bfloat16, 2, 200, 4, 4, 128, 0, 300, 100),   # group 1, R beyond T, temperature
    (torch.bfloat16, 1, 129, 4, 2, 128, 64, 32, 0),     # one tile plus one row, window < tile
    (torch.bfloat16, 1, 1024, 32, 4, 128, 512, 512, 0), # the local layer's 32 / 4 head layout
    (torch.bfloat16, 1, 700, 8, 2, 128, 512, 512, 300),  # window and temperature together
    (torch.bfloat16, 1, 2300, 4, 2, 128, 0, 2048, 0),    # the largest R, global layer, ragged tail
    (torch.bfloat16, 1, 600, 4, 2, 64, 200, 64, 0),      # d = 64, window not a tile multiple, R < window
]


@pytest.mark.parametrize("dtype,B,T,Hq,Hkv,d,window,R,temp_n0", CASES)
def test_backward_parity(dtype, B, T, Hq, Hkv, d, window, R, temp_n0):
    x = _inputs(dtype, B, T, Hq, Hkv, d, R, seed=T + d + R)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), window,
                                    R, scale, temp_n0=temp_n0)
    o = torch.as_tensor(o_ref).to(dtype).cuda()
    lse = torch.as_tensor(lse_ref).float().cuda()
    g = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], window, R, scale, temp_n0=temp_n0)
    torch.cuda.synchronize()
    ref = O.attn_backward(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), x["dout"].cpu(),
                          window, R, scale, temp_n0=temp_n0)
    _check(g, ref, 1e-4 if dtype == torch.float32 else 1e-2,
           "backward %s" % ((dtype, B, T, Hq, Hkv, d, window, R, temp_n0),))


def test_backward_after_the_bf16_forward():
    """A training step's own pair: the tensor-core forward's O and LSE feed the backward."""
    B, T, Hq, Hkv, d, window, R = 1, 640, 8, 2, 128, 512, 512
    x = _inputs(torch.bfloat16, B, T, Hq, Hkv, d, R, seed=3)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, lse=lse)
    g = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], window, R)
    torch.cuda.synchronize()
    ref = O.attn_backward(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), x["dout"].cpu(),
                          window, R, 1.0 / math.sqrt(d))
    _check(g, ref, 2e-2, "backward after forward")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_is_deterministic_except_dw(dtype):
    """dq, dk, dv and dr are written without atomics: bitwise repeatable."""
    x = _inputs(dtype, 1, 200, 4, 2, 64, 64, seed=11)
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["r"].cpu(), x["w"].cpu(), 0, 64,
                                    0.125)
    o = torch.as_tensor(o_ref).to(dtype).cuda()
    lse = torch.as_tensor(lse_ref).float().cuda()
    g1 = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], 0, 64, 0.125)
    g2 = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], 0, 64, 0.125)
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dr"):
        assert torch.equal(g1[name], g2[name]), name
    assert (g1["dw"] - g2["dw"]).abs().max().item() <= 1e-5 * g1["dw"].abs().max().item()


# The shared-bank form (relbias_attn_bwd_bank): bf16, d in {64, 128}.
BANK_CASES = [
    # B, T,   Hq, Hkv, d,   window, R,   C,  proj_heads, temp_n0
    (1, 300, 8, 2, 128, 0, 256, 16, 1, 0),       # the essay's 16-function bank, shared by the layer
    (1, 640, 8, 2, 128, 512, 512, 16, 8, 0),     # a bank per head, the local layer's window
    (2, 200, 6, 3, 64, 0, 150, 5, 1, 100),       # d = 64, odd group, R not a multiple of 8, temperature
    (1, 129, 4, 2, 128, 64, 30, 3, 4, 0),        # one tile plus one row, window < tile
    (1, 700, 4, 2, 128, 512, 512, 16, 1, 300),   # window and temperature together
    (1, 1300, 4, 2, 128, 0, 1024, 16, 1, 0),     # the global layer's R, ragged tail
]


def _bank_inputs(B, T, Hq, Hkv, d, R, C, proj_heads, seed):
    x = _inputs(torch.bfloat16, B, T, Hq, Hkv, d, R, seed)
    x["rs"] = synth.normal((B, T, Hq, C), seed, "rs", std=1.0 / math.sqrt(C), device="cuda")
    x["proj"] = synth.normal((proj_heads, C, R), seed, "proj", std=0.5, device="cuda")
    return x


@pytest.mark.parametrize("B,T,Hq,Hkv,d,window,R,C,proj_heads,temp_n0", BANK_CASES)
def test_backward_bank_parity(B, T, Hq, Hkv, d, window, R, C, proj_heads, temp_n0):
    """Gradients of the bank form (dq, dk, dv, drs, dproj) against the oracle's."""
    x = _bank_inputs(B, T, Hq, Hkv, d, R, C, proj_heads, seed=T + C + R)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = O.attn_prefill(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["rs"].cpu(), x["proj"].cpu(),
                                    window, R, scale, temp_n0=temp_n0)
    o = torch.as_tensor(o_ref).to(torch.bfloat16).cuda()
    lse = torch.as_tensor(lse_ref).float().cuda()
    g = ops.attn_bwd_bank(x["q"], x["k"], x["v"], x["rs"], x["proj"], o, lse, x["dout"], window, R, scale,
                          temp_n0=temp_n0)
    torch.cuda.synchronize()
    ref = O.attn_backward(x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), x["rs"].cpu(), x["proj"].cpu(),
                          x["dout"].cpu(), window, R, scale, temp_n0=temp_n0)
    _check({"dq": g["dq"], "dk": g["dk"], "dv": g["dv"], "dr": g["drs"], "dw": g["dproj"]}, ref, 1e-2,
           "bank backward %s" % ((B, T, Hq, Hkv, d, window, R, C, proj_heads, temp_n0),))


def test_backward_bank_of_one_function_per_head_matches_rank1():
    """C = 1 with a bank per head is the rank-1 form: the same gradients (drs = dr,
    dproj = dw) up to the order of the fp32 sums."""
    B, T, Hq, Hkv, d, window, R = 1, 400, 8, 2, 128, 256, 256
    x = _inputs(torch.bfloat16, B, T, Hq, Hkv, d, R, seed=21)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], window, R, lse=lse)
    g1 = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], window, R)
    g2 = ops.attn_bwd_bank(x["q"], x["k"], x["v"], x["r"][..., None].contiguous(), x["w"][:, None, :].contiguous(),
                           o, lse, x["dout"], window, R)
    torch.cuda.synchronize()
    for a, b in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dr", "drs"), ("dw", "dproj")):
        u, w = g1[a].reshape(-1), g2[b].reshape(-1)
        assert (u - w).abs().max().item() <= 1e-4 * u.abs().max().item() + 1e-7, a


@pytest.mark.parametrize("bank", [False, True])
def test_backward_full_size_local_layer_sampled(bank):
    """The local-layer workload at full size (B=2, T=8192, Hq=32, Hkv=4, d=128, window =
    R = 512, bf16), in the launch configuration the bench times.  A row's dq and dr
    depend only on the 512 keys it sees, and a key's dk and dv only on the 512 rows that
    see it, so the oracle over positions [i0 - 511, i0 + 64 + 511) of one sequence and
    one key/value head (with its 8 query heads) gives exact references for rows
    [i0, i0 + 64) (dq, dr: every key they see is in the slice) and
    keys [i0, i0 + 64) (dk, dv: every row that sees them is in the slice, with all of
    its own keys)."""
    from attention_learned_relative_b200 import workloads
    wl = workloads.WORKLOADS["local_backward_bf16"]
    x = workloads.make_inputs(wl, device="cuda")
    B, T, Hq, Hkv, d, W, R = wl.B, wl.T, wl.Hq, wl.Hkv, wl.d, wl.window, wl.R
    G = Hq // Hkv
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device="cuda")
    if bank:
        C = 16
        rs = synth.normal((B, T, Hq, C), 5, "rs", std=0.25, device="cuda")
        proj = synth.normal((1, C, R), 5, "proj", std=0.5, device="cuda")
        o = ops.attn_fwd_bank(x["q"], x["k"], x["v"], rs, proj, W, R, wl.scale, lse=lse)
        g = ops.attn_bwd_bank(x["q"], x["k"], x["v"], rs, proj, o, lse, x["dout"], W, R, wl.scale)
    else:
        o = ops.attn_fwd(x["q"], x["k"], x["v"], x["r"], x["w"], W, R, wl.scale, lse=lse)
        g = ops.attn_bwd(x["q"], x["k"], x["v"], x["r"], x["w"], o, lse, x["dout"], W, R, wl.scale)
    torch.cuda.synchronize()
    b, kv, i0, n = 1, 2, 5000, 64
    lo, hi = i0 - (W - 1), i0 + n + (W - 1)
    heads = slice(kv * G, (kv + 1) * G)
    sl = lambda t: t[b:b + 1, lo:hi].cpu()
    if bank:
        r_in, w_in = rs[b:b + 1, lo:hi, heads].cpu(), proj.cpu()
    else:
        r_in, w_in = x["r"][b:b + 1, lo:hi, heads].cpu(), x["w"][heads].cpu()
    ref = O.attn_backward(sl(x["q"])[:, :, heads], sl(x["k"])[:, :, kv:kv + 1], sl(x["v"])[:, :, kv:kv + 1], r_in, w_in,
                          sl(x["dout"])[:, :, heads], W, R, wl.scale)
    dr_name = "drs" if bank else "dr"
    checks = [
        ("dq", g["dq"][b, i0:i0 + n, heads].double().cpu(), torch.as_tensor(ref["dq"])[0, W - 1:W - 1 + n]),
        ("dr", g[dr_name][b, i0:i0 + n, heads].double().cpu(), torch.as_tensor(ref["dr"])[0, W - 1:W - 1 + n]),
        ("dk", g["dk"][b, i0:i0 + n, kv].double().cpu(), torch.as_tensor(ref["dk"])[0, W - 1:W - 1 + n, 0]),
        ("dv", g["dv"][b, i0:i0 + n, kv].double().cpu(), torch.as_tensor(ref["dv"])[0, W - 1:W - 1 + n, 0]),
    ]
    for name, got, want in checks:
        err = (got - want).abs().max().item()
        scale = want.abs().max().item()
        assert err <= 2e-2 * scale + 1e-7, "%s %s: max err %.3e vs max |ref| %.3e" % ("bank" if bank else "rank-1",
                                                                                     name, err, scale)
