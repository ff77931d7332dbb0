"""The multi-layer prefill's kernels through the C ABI against the fp64 layer oracle
(oracle/layer_oracle.py) and plain fp32 references.

* spava_qkv_projection (RMSNorm row scale + QKV GEMM + split into q/k/v) and
  spava_out_projection (GEMM + residual, in place) against fp32 references, on
  ragged row counts (not multiples of the 128-row tile) and several column tiles.
* One and three layers of LayerStack, each step of each layer against the oracle on
  the GPU's own inputs to that step: the projections within bf16 rounding of the
  fp64 result, the attention within the prefill's tolerances (max |dO| <= 2e-2,
  max |dlse| <= 1e-3) of the oracle re-run with the GPU's selection, the residual
  within bf16 rounding; and the whole stack against the oracle stack run in fp64
  from the same input with the GPU's selections.
* With one host the approximate and dense stacks agree; hidden states stay finite.

Tolerances: a bf16 result rounded to nearest is within 2^-9 of its value relative;
the fp32 accumulation over K <= 4096 products of exact bf16 values adds well under
1e-5 relative.  So projections are checked at |d| <= 2^-8 |y| + 1e-3 max|y|.  Over
the whole stack the roundings of q, k, v, o and x add up (about six roundings per
layer feed the next layer's input), checked at 4e-2 of max |x| per layer.
"""

import math

import numpy as np
import pytest
import torch

from oracle import layer_oracle as lo
from oracle import spava_oracle as orc
from workloads import CONFIGS, generate

from .helpers import LSE_TOL, O_TOL, make_plan

pytestmark = pytest.mark.gpu

sab = pytest.importorskip("sequence_approximate_attention_b200")

CFG = CONFIGS["tiny"].with_(n_visual=1024, n_hosts=4, head_dim=128, hq=4, hkv=2, anchor=64, passing=64,
                            probe_r=32, n_text=40, seed=21)
CFG_G7 = CONFIGS["tiny"].with_(n_visual=768, n_hosts=3, head_dim=128, hq=14, hkv=2, anchor=32, passing=96,
                               probe_r=32, n_text=17, seed=22)
EPS = 1e-6


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _proj_close(got: torch.Tensor, want: np.ndarray, what: str) -> None:
    g = _f64(got).reshape(want.shape)
    err = np.abs(g - want)
    tol = 2.0 ** -8 * np.abs(want) + 1e-3 * np.abs(want).max()
    assert (err <= tol).all(), (what, float(err.max()), float(np.abs(want).max()))


@pytest.mark.parametrize("M,hidden,hq,hkv", [(1000, 512, 4, 2), (257, 1792, 14, 2), (128, 256, 2, 2)])
def test_qkv_projection_against_fp32(M, hidden, hq, hkv):
    d = 128
    g = torch.Generator().manual_seed(M + hidden)
    x = (torch.randn(M, hidden, generator=g) * 0.7).to(torch.bfloat16).cuda()
    w = (torch.randn((hq + 2 * hkv) * d, hidden, generator=g) / math.sqrt(hidden)).to(torch.bfloat16).cuda()
    q = torch.full((M, hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    k = torch.full((M, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    v = torch.full((M, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = sab.layer_workspace(M)
    sab.qkv_projection(x, w, hq, hkv, d, q, k, v, ws, EPS)
    sab.check_layer_error(ws)
    xf = x.double()
    y = ((xf / torch.sqrt((xf * xf).mean(dim=1, keepdim=True) + EPS)) @ w.double().T).cpu().numpy()
    nq, nk = hq * d, hkv * d
    _proj_close(q, y[:, :nq], "q")
    _proj_close(k, y[:, nq:nq + nk], "k")
    _proj_close(v, y[:, nq + nk:], "v")


@pytest.mark.parametrize("M,in_f,hidden", [(1000, 512, 512), (300, 1792, 256)])
def test_out_projection_residual_against_fp32(M, in_f, hidden):
    g = torch.Generator().manual_seed(M + in_f)
    o = torch.randn(M, in_f, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(hidden, in_f, generator=g) / math.sqrt(in_f)).to(torch.bfloat16).cuda()
    x = torch.randn(M, hidden, generator=g).to(torch.bfloat16).cuda()
    want = (x.double() + o.double() @ w.double().T).cpu().numpy()
    ws = sab.layer_workspace(M)
    sab.out_projection(o, w, x, ws)
    sab.check_layer_error(ws)
    _proj_close(x, want, "x + o W_o^T")


def _stack(cfg, n_layers, seed=3):
    from sequence_approximate_attention_b200.layer_stack import LayerStack

    g = generate(cfg)
    plan = make_plan(sab, cfg, g["host_sizes"])
    hidden = cfg.hq * cfg.head_dim
    stack = LayerStack(plan, hidden, n_layers, seed=seed, rms_eps=EPS)
    x = (torch.randn(plan.n_total, hidden, generator=torch.Generator().manual_seed(seed + 1)) * 0.5)
    return g, plan, stack, x.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("cfg,n_layers", [(CFG, 1), (CFG, 3), (CFG_G7, 3)], ids=["1layer", "3layers", "g7_3layers"])
def test_layers_against_oracle(cfg, n_layers):
    g, plan, stack, x = _stack(cfg, n_layers)
    rec = []
    out = stack.forward(x, record=rec).clone()
    stack.check_errors()
    torch.cuda.synchronize()
    sizes = [int(s) for s in g["host_sizes"]]
    off = orc.host_offsets(sizes)
    d, hq, hkv = cfg.head_dim, cfg.hq, cfg.hkv
    scale = 1.0 / math.sqrt(d)
    NT = plan.n_total
    layers64 = [{"w_qkv": _f64(L["w_qkv"]), "w_o": _f64(L["w_o"])} for L in stack.layers]
    sels = []
    for li, r in enumerate(rec):
        L = layers64[li]
        # projections on the GPU's input to this layer
        x_in = _f64(r["x"])
        y = lo.rms_norm(x_in, EPS) @ L["w_qkv"].T
        nq, nk = hq * d, hkv * d
        _proj_close(r["q"], y[:, :nq].reshape(NT, hq, d), f"layer {li} q")
        _proj_close(r["k"], y[:, nq:nq + nk].reshape(NT, hkv, d), f"layer {li} k")
        _proj_close(r["v"], y[:, nq + nk:].reshape(NT, hkv, d), f"layer {li} v")
        # attention on the GPU's q/k/v with the GPU's selection (bit-exact given its scores
        # is covered by the prefill parity tests)
        sel = r["sel"].cpu().numpy().astype(np.int64)
        sels.append(sel)
        ref = orc.prefill(_f64(r["q"]), _f64(r["k"]), _f64(r["v"]), sizes, cfg.anchor, cfg.passing, cfg.probe_r,
                          scale=scale, sel=sel)
        do = np.abs(_f64(r["o"]) - ref["O"]).max()
        dl = np.abs(r["lse"].cpu().numpy() - ref["lse"]).max()
        assert do <= O_TOL and dl <= LSE_TOL, (li, do, dl)
        # output projection + residual on the GPU's o
        x_next = x_in + _f64(r["o"]).reshape(NT, nq) @ L["w_o"].T
        x_gpu = rec[li + 1]["x"] if li + 1 < len(rec) else out
        _proj_close(x_gpu, x_next, f"layer {li} residual")
    # the whole stack in fp64 from the same input, with the GPU's selections
    want = lo.attention_stack(_f64(x), layers64, hq, hkv, d, sizes, cfg.anchor, cfg.passing, cfg.probe_r, EPS,
                              sels=sels)[-1]["x"]
    err = np.abs(_f64(out) - want).max()
    assert err <= 4e-2 * n_layers * np.abs(want).max(), (err, np.abs(want).max())
    plan.close()


def test_one_host_stack_equals_dense():
    _, plan, stack, x = _stack(CFG.with_(n_hosts=1), 3)
    a = stack.forward(x).clone().float()
    b = stack.forward(x, dense=True).clone().float()
    stack.check_errors()
    torch.cuda.synchronize()
    assert torch.isfinite(a).all() and torch.isfinite(b).all()
    assert (a - b).abs().max().item() <= 5e-2 * max(1.0, b.abs().max().item())
    plan.close()


def test_stack_stays_finite():
    _, plan, stack, x = _stack(CFG, 4)
    y = stack.forward(x)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    assert stack.flops()["projections"] > 0
    plan.close()
