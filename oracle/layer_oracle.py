"""fp64 CPU oracle of the attention block of one decoder layer around the
approximate-attention prefill, for the multi-layer prefill.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and the CPU-baseline leg of
``bench.py``, never by the library, and it imports nothing from the library.

The pages report time to first token of whole long-video models (APB-V technical
summary, "Experimental results") and describe how the query segment's forward is
fused with the context's (2. System optimisations, "Fused context and query
forward"), but they define no layer.  Reading L1 (parity unpinned against the pages:
no page value fixes it): the attention block of a Qwen2-class decoder layer without
rotary embedding, norm gain or MLP, every token of the layer (visual and text) going
through the same maps:

    h        = x / sqrt(mean_j x_j^2 + eps)                (RMSNorm, per token)
    q | k | v = h W_qkv^T                                  (W_qkv = [W_q; W_k; W_v])
    o        = approximate-attention prefill of (q, k, v)  (spava_oracle.prefill)
    x'       = x + o W_o^T                                 (output projection, residual)

with q [tokens, hq, d] and k, v [tokens, hkv, d] taken as consecutive column blocks of
h W_qkv^T, and o read back as [tokens, hq d].  Everything is float64; weights and
inputs given as bf16 values are converted exactly by the caller.
"""

from typing import Dict, List, Optional, Sequence

import numpy as np

from . import spava_oracle as orc


def rms_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """Each row divided by the square root of (its mean square + eps)."""
    return x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)


def attention_block(x: np.ndarray, w_qkv: np.ndarray, w_o: np.ndarray, hq: int, hkv: int, head_dim: int,
                    host_sizes: Sequence[int], anchor: int, passing: int, probe_r: int, eps: float = 1e-6,
                    sel: Optional[np.ndarray] = None, scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """One attention block on x [tokens, hidden].  ``sel`` replaces the prefill's own
    selection (to re-run it with another one).  Returns the block's output x' and its
    intermediates q, k, v, O, lse and the selection used."""
    T = x.shape[0]
    nq, nk = hq * head_dim, hkv * head_dim
    if w_qkv.shape != (nq + 2 * nk, x.shape[1]):
        raise ValueError("w_qkv must be [(hq + 2 hkv) head_dim, hidden]")
    if w_o.shape != (x.shape[1], nq):
        raise ValueError("w_o must be [hidden, hq head_dim]")
    h = rms_norm(x, eps)
    y = np.matmul(h, w_qkv.T)
    q = y[:, :nq].reshape(T, hq, head_dim)
    k = y[:, nq:nq + nk].reshape(T, hkv, head_dim)
    v = y[:, nq + nk:].reshape(T, hkv, head_dim)
    res = orc.prefill(q, k, v, host_sizes, anchor, passing, probe_r, scale=scale, sel=sel)
    out = x + np.matmul(res["O"].reshape(T, nq), w_o.T)
    return {"x": out, "q": q, "k": k, "v": v, "O": res["O"], "lse": res["lse"], "sel": res["sel"]}


def attention_stack(x: np.ndarray, layers: Sequence[Dict[str, np.ndarray]], hq: int, hkv: int, head_dim: int,
                    host_sizes: Sequence[int], anchor: int, passing: int, probe_r: int, eps: float = 1e-6,
                    sels: Optional[Sequence[np.ndarray]] = None) -> List[Dict[str, np.ndarray]]:
    """Blocks applied in order (layers: dicts with w_qkv and w_o); the output of each
    is the input of the next.  ``sels[l]`` replaces layer l's selection."""
    out = []
    for li, L in enumerate(layers):
        r = attention_block(x, L["w_qkv"], L["w_o"], hq, hkv, head_dim, host_sizes, anchor, passing, probe_r, eps,
                            sel=None if sels is None else sels[li])
        out.append(r)
        x = r["x"]
    return out
