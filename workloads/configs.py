"""The five synthetic workloads of the approximate-attention prefill.

Each one is a single attention layer of a long-video LMM prefill: N visual tokens
split into H contiguous host blocks, an anchor of A tokens, P passing keys per
host and KV head, R probe queries per host, GQA heads (hq query / hkv KV heads,
head_dim d) and an optional trailing text segment of T tokens that attends
densely.  Head counts and head_dim follow Qwen2-class layers (28/4 or 32/8
heads, d=128) and 256-token video frames, the model family the Spava / APB-V
pages evaluate (APB-V technical summary, "Experimental results").
"""

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    n_visual: int            # N
    n_hosts: int             # H
    anchor: int              # A
    passing: int             # P
    probe_r: int             # R
    hq: int
    hkv: int
    head_dim: int
    n_text: int = 0          # T
    kv_kind: str = "iid"     # "iid" | "frame"
    frame: int = 256         # tokens per video frame (frame-built K/V)
    frame_noise: float = 0.3
    salient_frac: float = 0.0
    salient_scale: float = 3.0
    uneven: Optional[Tuple[int, int, int]] = None   # (min, max, multiple) block sizes
    seed: int = 0
    description: str = field(default="", compare=False)

    @property
    def n_total(self) -> int:
        return self.n_visual + self.n_text

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


CONFIGS = {
    "tiny": Workload(
        name="tiny", n_visual=512, n_hosts=2, anchor=64, passing=32, probe_r=16,
        hq=4, hkv=2, head_dim=64, n_text=0, kv_kind="iid", seed=0,
        description="N=512, H=2x256, A=64, P=32, R=16, 4/2 heads, d=64, iid N(0,1)"),
    "qwen64k": Workload(
        name="qwen64k", n_visual=65536, n_hosts=8, anchor=2048, passing=1024, probe_r=64,
        hq=28, hkv=4, head_dim=128, n_text=128, kv_kind="frame", seed=1,
        description="Qwen2-VL-7B-like layer: N=65536, H=8x8192, A=2048, P=1024, R=64, "
                    "28/4 heads, d=128, frame-built K/V, 128 text tokens"),
    "128k": Workload(
        name="128k", n_visual=131072, n_hosts=16, anchor=4096, passing=1024, probe_r=64,
        hq=32, hkv=8, head_dim=128, n_text=256, kv_kind="frame", salient_frac=0.05, seed=2,
        description="N=131072 (512 frames x 256), H=16x8192, A=4096, P=1024, R=64, "
                    "32/8 heads, d=128, frame-built K/V + 5% salient keys x3, 256 text tokens"),
    "stress": Workload(
        name="stress", n_visual=131072, n_hosts=16, anchor=2048, passing=2048, probe_r=128,
        hq=28, hkv=4, head_dim=128, n_text=0, kv_kind="iid", uneven=(4096, 12288, 64), seed=3,
        description="load-balance stress: N=131072 in 16 uneven blocks (4096..12288), "
                    "A=2048, P=2048, R=128, 28/4 heads, d=128, iid N(0,1)"),
    "256k": Workload(
        name="256k", n_visual=262144, n_hosts=32, anchor=4096, passing=512, probe_r=64,
        hq=32, hkv=8, head_dim=128, n_text=256, kv_kind="frame", seed=4,
        description="N=262144 (1024 frames x 256), H=32x8192, A=4096, P=512, R=64, "
                    "32/8 heads, d=128, frame-built K/V, 256 text tokens"),
}


def get_config(name: str) -> Workload:
    try:
        return CONFIGS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}") from None
