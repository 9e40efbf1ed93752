"""GPU checks of the decode option ``independent_state`` (``rwkv7_options``): the state loads of a step
start before the wait for the step before it on the stream, which the caller allows when no step still
running writes that state.  A model with several layers, each keeping its own state and stepped in
turn, is that case; the recurrence is the x070 single-step update of the RWKV-7 G0 7.2B walkthrough
(lshu.cn/news/198401), section 7.1.

The option changes only when the loads are issued, not the arithmetic.  So a run of steps over
rotating layer states with the option set must give bit-for-bit the same outputs and states as the
same run without it.  That holds for the float32 state (bf16 operands, model-native inputs, the
GroupNorm epilogue) and for the bf16 state, on a stream and replayed from a CUDA graph.  The run
without the option is itself checked against the float64 oracle by the other decode tests; its
first layer's first step is checked here too.  The shape, B256 H16 with three layer states, keeps
every grid larger than the device runs at once, where the option takes effect; a last test checks
that smaller steps ignore it.
"""

import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, rel_err

pytestmark = pytest.mark.gpu

B, H, N, LAYERS, STEPS = 256, 16, 64, 3, 12
NATIVE = ("r", "xw", "k", "v", "xa")


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _tokens(native, seed):
    dev = torch.device("cuda", 0)
    if native:
        d = wi.draw_model_native(B, STEPS, H, seed=seed, device=dev)
        names = NATIVE
    else:
        d = wi.draw(B, STEPS, H, seed=seed, dtype="bf16", device=dev, f32_copies=False)
        names = OPS
    toks = {n: d[n].transpose(0, 1).contiguous() for n in names}  # [STEPS, B, H, N]
    return toks, (d["k_k"] if native else None)


def _run(mode, independent, graph, seed=71):
    """STEPS decode steps over LAYERS rotating states; returns (ys, states)."""
    native, gn, bf16 = mode == "native", mode == "group_norm", mode == "bf16_state"
    toks, kk = _tokens(native, seed)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    s0 = (torch.randn(LAYERS, B, H, N, N, generator=g) * 0.1).to(dev)
    states = s0.to(torch.bfloat16) if bf16 else s0.clone()
    ln = {k: t.to(dev) for k, t in wi.draw_group_norm(H, seed=seed + 2).items()} if gn else {}
    ys = torch.empty(STEPS, B, H, N, dtype=torch.bfloat16, device=dev)
    names = NATIVE if native else OPS

    def one_pass():
        for i in range(STEPS):
            L = i % LAYERS
            ops = [toks[n][i] for n in names] + ([None] if native else [])
            if bf16:
                rk.rwkv7_wkv_decode_ext_bf16state(*ops, states[L], ys[i], independent_state=independent)
            else:
                rk.rwkv7_wkv_decode_ext_bf16(*ops, states[L], ys[i], model_native=native, k_k=kk, group_norm=gn,
                                             ln_w=ln.get("ln_w"), ln_b=ln.get("ln_b"),
                                             independent_state=independent)

    if graph:
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=s):
            one_pass()
        cg.replay()
    else:
        one_pass()
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    first = {n: toks[n][0].cpu() for n in names}
    return ys.cpu(), states.float().cpu(), first, s0.cpu(), kk, ln


MODES = ["f32_state", "native", "group_norm", "bf16_state"]


@pytest.mark.parametrize("graph", [False, True], ids=["stream", "graph"])
@pytest.mark.parametrize("mode", MODES)
def test_independent_state_gives_the_same_bits(mode, graph):
    y0, s0, *_ = _run(mode, False, graph)
    y1, s1, *_ = _run(mode, True, graph)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert torch.equal(s0, s1)


@pytest.mark.parametrize("mode", ["f32_state", "native"])
def test_first_step_matches_the_oracle(mode):
    """Step 0 (layer 0) of the run with the option set, against the float64 step."""
    ys, _, first, s0, kk, _ = _run(mode, True, False)
    if mode == "native":
        f32 = {n: first[n].float() for n in NATIVE}
        yo, _ = oracle.wkv7_model_native(*[f32[n][:, None] for n in NATIVE], kk.cpu(), s0[0])
    else:
        f32 = {n: first[n].float() for n in OPS}
        yo, _ = oracle.wkv7(*[f32[n][:, None] for n in OPS], s0[0])
    assert rel_err(ys[0], yo[:, 0]) <= TOL_BF16


@pytest.mark.parametrize("bf16", [False, True], ids=["f32_state", "bf16_state"])
def test_small_steps_ignore_the_option(bf16):
    """Below the device's resident CTA count the library keeps the wait before the state loads, so even
    steps that violate the promise (every step on one state, B1 H4) stay exact: bit-for-bit the same
    as without the option."""
    b, h, steps = 1, 4, 16
    dev = torch.device("cuda", 0)
    d = wi.draw(b, steps, h, seed=91, dtype="bf16", device=dev, f32_copies=False)
    toks = {n: d[n].transpose(0, 1).contiguous() for n in OPS}
    g = torch.Generator(device="cpu").manual_seed(92)
    s_init = (torch.randn(b, h, N, N, generator=g) * 0.1).to(dev)
    out = []
    for independent in (False, True):
        state = s_init.to(torch.bfloat16) if bf16 else s_init.clone()
        ys = torch.empty(steps, b, h, N, dtype=torch.bfloat16, device=dev)
        for i in range(steps):
            ops = [toks[n][i] for n in OPS]
            if bf16:
                rk.rwkv7_wkv_decode_ext_bf16state(*ops, state, ys[i], independent_state=independent)
            else:
                rk.rwkv7_wkv_decode_ext_bf16(*ops, state, ys[i], independent_state=independent)
        torch.cuda.synchronize()
        out.append((ys.cpu(), state.float().cpu()))
    assert torch.equal(out[0][0].view(torch.int16), out[1][0].view(torch.int16))
    assert torch.equal(out[0][1], out[1][1])
